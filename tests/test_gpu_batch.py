"""GPU parity of bonsai_lowbit_gemm_batch: several independent GEMMs in one
call, every problem compared with the CPU oracle through the C ABI.

- mixed batches of ragged shapes (1..16 tokens, N not a multiple of 128,
  K from one group to 24), every output, in every storage format, with
  larger-M, K = 0 and empty problems among them;
- more problems than one launch takes (so the batch is cut in two);
- scales with negatives, signed zeros, subnormals and large magnitudes;
- the 80 linears of one denoise step at 16 tokens in one call, in every
  storage format, and 80 MLP-down layers (3072x9216) at 16 tokens, as the
  benchmark times them;
- a batch captured in a CUDA graph and replayed.

Bar as everywhere: |gpu - oracle| <= 1e-3 * sum_k |a_k w_k| + one FP16 ulp
of the oracle value, infinities and NaN matched in kind.
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


def build(oracle_mod, mode, shapes, seed0):
    """-> host arrays and device tensors of one problem per (M, N, K)."""
    probs = []
    for j, (M, N, K) in enumerate(shapes):
        d = workloads.make(mode=mode, M=M, N=N, K=K, seed=seed0 + j)
        probs.append({
            "d": d,
            "ref_packed": oracle_mod.pack(d["codes"], mode),
            "A": dev(d["A"].view(np.int16), torch.float16),
            "packed": bw.pack(dev(d["codes"]), mode),
            "s": dev(d["scales"].view(np.int16), torch.float16),
        })
    torch.cuda.synchronize()
    return probs


def check_all(oracle_mod, mode, probs, outs, label):
    for j, (p, out) in enumerate(zip(probs, outs)):
        d = p["d"]
        if d["M"] == 0 or d["N"] == 0:
            continue
        ref, _, absacc = oracle_mod.gemm(d["A"], p["ref_packed"], d["scales"], d["K"], mode)
        check(oracle_mod, to_u16(out), ref, absacc, f"{label} problem {j} {d['M']}x{d['N']}x{d['K']}")


MIXED = [(16, 256, 640), (1, 128, 128), (7, 1000, 1152), (16, 384, 3072), (3, 8, 128), (12, 2056, 384),
         (16, 136, 512), (40, 256, 512), (9, 512, 256), (16, 1280, 1536), (2, 648, 2048), (5, 96, 896)]


@pytest.mark.parametrize("mode", MODES)
def test_mixed_batch_every_output(oracle_mod, mode):
    probs = build(oracle_mod, mode, MIXED, 7000)
    outs = bw.lowbit_gemm_batch([(p["A"], p["packed"], p["s"]) for p in probs], mode)
    torch.cuda.synchronize()
    check_all(oracle_mod, mode, probs, outs, f"{mode} mixed batch")


def test_batch_with_empty_and_k0_problems(oracle_mod):
    """K = 0 problems get zeros; M = 0 and N = 0 problems are skipped; the
    others are computed."""
    mode = "ternary"
    probs = build(oracle_mod, mode, [(16, 256, 512), (4, 128, 256)], 7100)
    A0 = torch.empty((5, 0), dtype=torch.float16, device="cuda")
    P0 = torch.empty((24, 0), dtype=torch.int32, device="cuda")
    S0 = torch.empty((24, 0), dtype=torch.float16, device="cuda")
    out_k0 = torch.full((5, 24), float("nan"), dtype=torch.float16, device="cuda")
    outs = bw.lowbit_gemm_batch(
        [(probs[0]["A"], probs[0]["packed"], probs[0]["s"]), (A0, P0, S0),
         (torch.empty((0, 256), dtype=torch.float16, device="cuda"), probs[1]["packed"], probs[1]["s"]),
         (probs[1]["A"], probs[1]["packed"], probs[1]["s"])],
        mode, outs=[torch.empty((16, 256), dtype=torch.float16, device="cuda"), out_k0,
                    torch.empty((0, 128), dtype=torch.float16, device="cuda"),
                    torch.empty((4, 128), dtype=torch.float16, device="cuda")])
    torch.cuda.synchronize()
    assert (to_u16(out_k0) == 0).all()
    check_all(oracle_mod, mode, probs, [outs[0], outs[3]], "batch with empty problems")


@pytest.mark.parametrize("mode", MODES)
def test_batch_larger_than_one_launch(oracle_mod, mode):
    """100 problems: more than one persistent launch takes, so two launches;
    1 to 5 groups per row, so word stages both whole and ragged."""
    shapes = [(1 + j % 16, 8 * (1 + j % 40), 128 * (1 + j % 5)) for j in range(100)]
    probs = build(oracle_mod, mode, shapes, 7200 + MODES.index(mode))
    outs = bw.lowbit_gemm_batch([(p["A"], p["packed"], p["s"]) for p in probs], mode)
    torch.cuda.synchronize()
    check_all(oracle_mod, mode, probs, outs, "100-problem batch")


F16_SPECIAL = [0x0000, 0x8000, 0x0001, 0x8001, 0x03FF, 0x0400, 0x8400, 0x3C00, 0xBC00, 0x77FF, 0xF7FF]


@pytest.mark.parametrize("mode", MODES)
def test_batch_special_scales(oracle_mod, mode):
    """Scales of random sign with signed zeros, subnormals and magnitudes up
    to the largest below 32768 on whole rows and single groups."""
    shapes = [(16, 640, 3072), (5, 136, 1152)]
    probs = build(oracle_mod, mode, shapes, 7300)
    rng = np.random.default_rng(7301)
    for p in probs:
        d = p["d"]
        N, G = d["N"], d["K"] // 128
        s = (rng.uniform(0.005, 0.05, (N, G)) * np.where(rng.random((N, G)) < 0.5, -1.0, 1.0)).astype(np.float16)
        s = s.view(np.uint16)
        for i, v in enumerate(F16_SPECIAL):
            s[(7 * i + 3) % N, :] = v
            s[(11 * i + 5) % N, (3 * i) % G] = v
        d["scales"] = s
        p["s"] = dev(s.view(np.int16), torch.float16)
    outs = bw.lowbit_gemm_batch([(p["A"], p["packed"], p["s"]) for p in probs], mode)
    torch.cuda.synchronize()
    check_all(oracle_mod, mode, probs, outs, f"{mode} batch special scales")


def _positions(M, N, count, seed):
    rng = np.random.default_rng(seed)
    ms = list(rng.integers(0, M, count))
    ns = list(rng.integers(0, N, count))
    for n in sorted({0, N - 1} | {x for b in range(128, N, 128) for x in (b - 1, b)}):
        ms += list(rng.integers(0, M, 2))
        ns += [n] * 2
    return np.array(ms, np.int64), np.array(ns, np.int64)


def _layers(oracle_mod, shapes, M, seed, distinct_codes=4, mode="ternary"):
    """Problems of the given (N, K) at M tokens: own activations and scales
    each, codes shared among every distinct_codes-th layer of a shape."""
    codes = {}
    rng = np.random.default_rng(seed)
    probs = []
    for j, (n, k) in enumerate(shapes):
        key = (n, k, j % distinct_codes)
        if key not in codes:
            d = workloads.make(mode=mode, M=1, N=n, K=k, seed=seed + 1 + len(codes))
            codes[key] = (bw.pack(dev(d["codes"]), mode), oracle_mod.pack(d["codes"], mode))
        a = workloads.activations(rng, M, k)
        s = workloads.scales(rng, n, k)
        probs.append({"a": a, "s_np": s, "A": dev(a.view(np.int16), torch.float16), "packed": codes[key][0],
                      "ref_packed": codes[key][1], "s": dev(s.view(np.int16), torch.float16), "N": n, "K": k})
    torch.cuda.synchronize()
    return probs


def _check_sampled(oracle_mod, probs, outs, M, label, full=(), mode="ternary"):
    for j, (p, out) in enumerate(zip(probs, outs)):
        got = to_u16(out)
        assert not np.isnan(got.view(np.float16)).any(), f"{label} {j}: an output was not written"
        if j in full:
            ref, _, absacc = oracle_mod.gemm(p["a"], p["ref_packed"], p["s_np"], p["K"], mode)
            check(oracle_mod, got, ref, absacc, f"{label} {j} (every output)")
            continue
        ms, ns = _positions(M, p["N"], 300, j)
        ref, _, absacc = oracle_mod.gemm_entries(p["a"], p["ref_packed"], p["s_np"], p["K"], mode, ms, ns)
        check(oracle_mod, got[ms, ns], ref, absacc, f"{label} {j}")


@pytest.mark.parametrize("mode", MODES)
def test_denoise_step_linears_at_16_tokens(oracle_mod, mode):
    """The 80 linears of one denoise step (Q|K|V stacked) at 16 tokens, in
    one call: one persistent launch over 2592 weight tiles, in every storage
    format (binary: 8 groups per word stage, two-turn slots of 48 KB;
    base-3: 112-byte blocks)."""
    layers = workloads.mmdit_stack_layers()
    probs = _layers(oracle_mod, [(n, k) for _, n, k in layers], 16, 7400 + MODES.index(mode), mode=mode)
    outs = [torch.full((16, p["N"]), float("nan"), dtype=torch.float16, device="cuda") for p in probs]
    bw.lowbit_gemm_batch([(p["A"], p["packed"], p["s"]) for p in probs], mode, outs=outs)
    torch.cuda.synchronize()
    # every output of one layer of each shape, sampled positions of the rest
    first = {}
    for j, p in enumerate(probs):
        first.setdefault((p["N"], p["K"]), j)
    _check_sampled(oracle_mod, probs, outs, 16, f"{mode} denoise-step linear", full=set(first.values()),
                   mode=mode)


def test_mlp_down_batch_at_16_tokens(oracle_mod):
    """80 MLP-down layers (3072x9216) at 16 tokens in one call, the
    benchmark's batched configuration."""
    probs = _layers(oracle_mod, [(3072, 9216)] * 80, 16, 7500)
    outs = [torch.full((16, 3072), float("nan"), dtype=torch.float16, device="cuda") for _ in probs]
    bw.lowbit_gemm_batch([(p["A"], p["packed"], p["s"]) for p in probs], "ternary", outs=outs)
    torch.cuda.synchronize()
    _check_sampled(oracle_mod, probs, outs, 16, "MLP-down batch", full={0, 79})


def test_batch_graph_replay(oracle_mod):
    """A batch captured in a CUDA graph and replayed twice, behind a plain
    GEMM in the same stream (the batch's weights are read while it runs)."""
    mode = "ternary"
    probs = build(oracle_mod, mode, [(16, 3072, 1536), (8, 1024, 3072), (16, 384, 512)], 7600)
    pre = build(oracle_mod, mode, [(256, 512, 1024)], 7650)[0]
    outs = [torch.empty((p["d"]["M"], p["d"]["N"]), dtype=torch.float16, device="cuda") for p in probs]
    pre_out = torch.empty((256, 512), dtype=torch.float16, device="cuda")

    def run():
        bw.lowbit_gemm(pre["A"], pre["packed"], pre["s"], mode, out=pre_out)
        bw.lowbit_gemm_batch([(p["A"], p["packed"], p["s"]) for p in probs], mode, outs=outs)

    run()
    torch.cuda.synchronize()
    for o in outs:
        o.fill_(float("nan"))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    del graph
    check_all(oracle_mod, mode, probs, outs, "graph-replayed batch")
    check_all(oracle_mod, mode, [pre], [pre_out], "GEMM before the batch")
