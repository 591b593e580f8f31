"""GPU parity at the configurations' full sizes and on special scales: every
output compared with the CPU oracle, through the C ABI.

- the two M=16 layers (MLP-down 3072x9216 and fused QKV 9216x3072) in every
  storage format and with the 4-bit group-affine weights, all outputs;
- one M=4608 layer (MLP-up 9216x3072) per format, all outputs (the oracle's
  double sums run threaded over the host's cores);
- GEMMs whose scales include negatives, signed zeros, subnormals and the
  largest magnitudes each format allows, over the one-tile, split-K and
  persistent launches;
- the single-stream layer shapes of the MMDiT stack (18432x3072 and
  3072x12288) at 4608 and 1536 tokens;
- one denoise step of the 80-launch stack replayed from a CUDA graph, every
  layer's output checked.

Bar as in test_gpu_parity: |gpu - oracle| <= 1e-3 * sum_k |a_k w_k| +
one FP16 ulp of the oracle value, infinities and NaN matched in kind.
"""
import numpy as np
import pytest
import torch

import bit_weight_gemm_b200 as bw
import workloads

pytestmark = pytest.mark.gpu

RTOL = 1e-3
MODES = ["binary", "ternary", "ternary_b3"]


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


def check(oracle_mod, got, ref, absacc, label):
    ok = oracle_mod.within_tolerance(got, ref, absacc, RTOL)
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        g = oracle_mod.half_bits_to_double(got)
        r = oracle_mod.half_bits_to_double(ref)
        details = [(tuple(i), g[tuple(i)], r[tuple(i)], absacc[tuple(i)]) for i in idx]
        pytest.fail(f"{label}: {int((~ok).sum())} of {ok.size} outside tolerance, e.g. {details}")


def run_case(oracle_mod, d, mode):
    packed_ref = oracle_mod.pack(d["codes"], mode)
    packed = bw.pack(dev(d["codes"]), mode)
    A = dev(d["A"].view(np.int16), torch.float16)
    s = dev(d["scales"].view(np.int16), torch.float16)
    out = bw.lowbit_gemm(A, packed, s, mode)
    torch.cuda.synchronize()
    ref, _, absacc = oracle_mod.gemm(d["A"], packed_ref, d["scales"], d["K"], mode)
    return to_u16(out), ref, absacc


# ----------------------------------------------------------- M = 16, full
SMALL_M = [workloads.TERNARY_MLP_DOWN_16, workloads.TERNARY_QKV_16]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("problem", SMALL_M, ids=[p.name for p in SMALL_M])
def test_small_m_every_output(oracle_mod, problem, mode):
    d = workloads.make(mode=mode, M=problem.M, N=problem.N, K=problem.K, seed=problem.seed)
    got, ref, absacc = run_case(oracle_mod, d, mode)
    check(oracle_mod, got, ref, absacc, f"{mode} {problem.name}")


@pytest.mark.parametrize("problem", SMALL_M, ids=[p.name for p in SMALL_M])
def test_small_m_every_output_hqq4(oracle_mod, problem):
    d = workloads.make_hqq4(problem.M, problem.N, problem.K, seed=problem.seed)
    packed = bw.hqq4_pack(dev(d["q"]))
    out = bw.hqq4_gemm(dev(d["A"].view(np.int16), torch.float16), packed, dev(d["scales"].view(np.int16), torch.float16),
                       dev(d["zeros"].view(np.int16), torch.float16))
    torch.cuda.synchronize()
    ref, _, absacc = oracle_mod.hqq4_gemm(d["A"], oracle_mod.hqq4_pack(d["q"]), d["scales"], d["zeros"], problem.K)
    check(oracle_mod, to_u16(out), ref, absacc, f"hqq4 {problem.name}")


# --------------------------------------------------------- M = 4608, full
@pytest.mark.parametrize("mode", MODES)
def test_large_m_every_output(oracle_mod, mode):
    p = workloads.TERNARY_MLP_UP_4608
    d = workloads.make(mode=mode, M=p.M, N=p.N, K=p.K, seed=p.seed)
    got, ref, absacc = run_case(oracle_mod, d, mode)
    check(oracle_mod, got, ref, absacc, f"{mode} {p.name}")


def test_large_m_every_output_hqq4(oracle_mod):
    p = workloads.TERNARY_MLP_UP_4608
    d = workloads.make_hqq4(p.M, p.N, p.K, seed=p.seed)
    packed = bw.hqq4_pack(dev(d["q"]))
    out = bw.hqq4_gemm(dev(d["A"].view(np.int16), torch.float16), packed, dev(d["scales"].view(np.int16), torch.float16),
                       dev(d["zeros"].view(np.int16), torch.float16))
    torch.cuda.synchronize()
    ref, _, absacc = oracle_mod.hqq4_gemm(d["A"], oracle_mod.hqq4_pack(d["q"]), d["scales"], d["zeros"], p.K)
    check(oracle_mod, to_u16(out), ref, absacc, f"hqq4 {p.name}")


# -------------------------------------------------------- special scales
F16 = {
    "+0": 0x0000, "-0": 0x8000, "min subnormal": 0x0001, "-min subnormal": 0x8001, "max subnormal": 0x03FF,
    "min normal": 0x0400, "-min normal": 0x8400, "1": 0x3C00, "-1": 0xBC00, "largest below 32768": 0x77FF,
    "-largest below 32768": 0xF7FF, "largest finite": 0x7BFF, "-largest finite": 0xFBFF,
}


def special_scales(rng, N, groups, mode):
    """Scales of random sign drawn from the workload's range, with every
    special value above placed on whole rows and on single groups.  The
    INT2 kernel's precondition is |s| < 32768, so only binary and base-3
    weights get the largest finite magnitude."""
    mag = rng.uniform(0.005, 0.05, (N, groups))
    s = (mag * np.where(rng.random((N, groups)) < 0.5, -1.0, 1.0)).astype(np.float16).view(np.uint16)
    specials = [v for k, v in F16.items() if mode != "ternary" or "finite" not in k]
    for i, v in enumerate(specials):
        s[(7 * i + 3) % N, :] = v                      # a whole row
        s[(11 * i + 5) % N, (3 * i) % groups] = v      # a single group
    return s


SPECIAL_SHAPES = [(40, 384, 512), (16, 640, 3072), (300, 1000, 1152), (1357, 3880, 512)]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M,N,K", SPECIAL_SHAPES)
def test_gemm_special_scales(oracle_mod, mode, M, N, K):
    d = workloads.make(mode=mode, M=M, N=N, K=K, seed=5 * M + N + K)
    rng = np.random.default_rng(M + N + K)
    d["scales"] = special_scales(rng, N, K // 128, mode)
    got, ref, absacc = run_case(oracle_mod, d, mode)
    r = ref.view(np.float16)
    assert np.isfinite(r).mean() > 0.5  # most rows stay finite: the case tests values, not only overflow
    check(oracle_mod, got, ref, absacc, f"{mode} special scales {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", SPECIAL_SHAPES)
def test_hqq4_special_scales_and_zeros(oracle_mod, M, N, K):
    """Scales and zeros with signed zeros, subnormals, negatives and large
    magnitudes, kept where every weight fp16(fp16(q - z) * s) is finite
    (|q - z| <= 31, |s| <= 2000)."""
    d = workloads.make_hqq4(M, N, K, seed=M + 2 * N + K)
    rng = np.random.default_rng(N + K)
    G = K // 64
    s = (rng.uniform(0.005, 0.05, (N, G)) * np.where(rng.random((N, G)) < 0.5, -1.0, 1.0)).astype(np.float16)
    z = rng.uniform(-16.0, 31.0, (N, G)).astype(np.float16)
    s, z = s.view(np.uint16), z.view(np.uint16)
    svals = [0x0000, 0x8000, 0x0001, 0x8001, 0x03FF, 0x0400, 0xBC00, np.float16(2000.0).view(np.uint16),
             np.float16(-1999.0).view(np.uint16)]
    zvals = [0x0000, 0x8000, 0x0001, 0x83FF, np.float16(-16.0).view(np.uint16), np.float16(31.0).view(np.uint16),
             np.float16(7.5).view(np.uint16)]
    for i, v in enumerate(svals):
        s[(5 * i + 1) % N, :] = v
        s[(13 * i + 2) % N, (7 * i) % G] = v
    for i, v in enumerate(zvals):
        z[(3 * i + 4) % N, :] = v
        z[(17 * i + 9) % N, (5 * i) % G] = v
    out = bw.hqq4_gemm(dev(d["A"].view(np.int16), torch.float16), bw.hqq4_pack(dev(d["q"])),
                       dev(s.view(np.int16), torch.float16), dev(z.view(np.int16), torch.float16))
    torch.cuda.synchronize()
    ref, _, absacc = oracle_mod.hqq4_gemm(d["A"], oracle_mod.hqq4_pack(d["q"]), s, z, K)
    check(oracle_mod, to_u16(out), ref, absacc, f"hqq4 special scales and zeros {M}x{N}x{K}")


# ------------------------------------------------- stack layer shapes
def _positions(M, N, count, seed):
    """Random positions plus every 128-row and 256-token tile edge, the first
    and last rows and columns."""
    rng = np.random.default_rng(seed)
    ms = list(rng.integers(0, M, count))
    ns = list(rng.integers(0, N, count))
    for m in sorted({0, M - 1} | {x for b in range(256, M, 256) for x in (b - 1, b)}):
        ms += [m] * 6
        ns += list(rng.integers(0, N, 6))
    for n in sorted({0, N - 1} | {x for b in range(128, N, 128) for x in (b - 1, b)}):
        ms += list(rng.integers(0, M, 2))
        ns += [n] * 2
    return np.array(ms, np.int64), np.array(ns, np.int64)


@pytest.mark.parametrize("M", [4608, 1536])
@pytest.mark.parametrize("N,K", [(18432, 3072), (3072, 12288)])
def test_single_stream_layer_shapes(oracle_mod, M, N, K):
    d = workloads.make(mode="ternary", M=M, N=N, K=K, seed=M + N + K)
    packed_ref = oracle_mod.pack(d["codes"], "ternary")
    out = bw.lowbit_gemm(dev(d["A"].view(np.int16), torch.float16), bw.pack(dev(d["codes"]), "ternary"),
                         dev(d["scales"].view(np.int16), torch.float16), "ternary")
    got = to_u16(out)
    ms, ns = _positions(M, N, 4000, M * 7 + N)
    ref, _, absacc = oracle_mod.gemm_entries(d["A"], packed_ref, d["scales"], K, "ternary", ms, ns)
    check(oracle_mod, got[ms, ns], ref, absacc, f"stack layer {M}x{N}x{K}")
    # whole rows at the start, the middle and the end of the token range
    rows = np.array([0, M // 2, M - 1])
    ref_rows, _, abs_rows = oracle_mod.gemm(d["A"][rows], packed_ref, d["scales"], K, "ternary")
    check(oracle_mod, got[rows], ref_rows, abs_rows, f"stack layer {M}x{N}x{K}, whole rows")


def test_graph_replayed_denoise_step(oracle_mod):
    """One denoise step (80 launches, Q|K|V stacked) at M=1024, captured in a
    CUDA graph and replayed twice; every layer has its own activations and
    scales (codes per distinct shape), and each layer's output is checked at
    sampled positions after the second replay."""
    M = 1024
    layers = workloads.mmdit_stack_layers()
    shapes = sorted({(n, k) for _, n, k in layers})
    codes = {}
    for j, (n, k) in enumerate(shapes):
        d = workloads.make(mode="ternary", M=1, N=n, K=k, seed=4000 + j)
        codes[(n, k)] = (d["codes"], bw.pack(dev(d["codes"]), "ternary"), oracle_mod.pack(d["codes"], "ternary"))
    rng = np.random.default_rng(4100)
    bufs = []
    for name, n, k in layers:
        a = workloads.activations(rng, M, k)
        s = workloads.scales(rng, n, k)
        bufs.append((a, s, dev(a.view(np.int16), torch.float16), dev(s.view(np.int16), torch.float16),
                     torch.empty((M, n), dtype=torch.float16, device="cuda")))
    torch.cuda.synchronize()

    def step():
        for (name, n, k), (_, _, A, s, out) in zip(layers, bufs):
            bw.lowbit_gemm(A, codes[(n, k)][1], s, "ternary", out=out)

    step()  # kernel attributes and tensor maps before capture
    torch.cuda.synchronize()
    for _, _, _, _, out in bufs:
        out.fill_(float("nan"))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    del graph
    for i, ((name, n, k), (a, s, _, _, out)) in enumerate(zip(layers, bufs)):
        got = to_u16(out)
        ms, ns = _positions(M, n, 300, i)
        ref, _, absacc = oracle_mod.gemm_entries(a, codes[(n, k)][2], s, k, "ternary", ms, ns)
        check(oracle_mod, got[ms, ns], ref, absacc, f"denoise step layer {i} {name}")
        assert not np.isnan(got.view(np.float16)).any(), f"layer {i} {name}: an output was not written"
