"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/bonsai.h declares, and rejects bad arguments before
touching a device.  Also checks that the CUDA side and the oracle stay
independent."""
import os
import re
import subprocess

import pytest

import bit_weight_gemm_b200 as bw
from bit_weight_gemm_b200 import build as bw_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bonsai.h")


@pytest.fixture(scope="module")
def lib():
    bw_build.build()
    return bw.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bonsai_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ["bonsai_pack", "bonsai_dequant", "bonsai_lowbit_gemm", "bonsai_lowbit_gemm_host",
                     "bonsai_lowbit_gemm_batch",
                     "bonsai_get_device_error",
                     "bonsai_status_string", "bonsai_packed_bytes", "bonsai_scale_bytes"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", bw.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (bonsai_\w+)", out))
    declared = set(declared_functions())
    assert declared <= exported, declared - exported
    assert declared == set(bw.SIGNATURES), "binding and header disagree"
    for name in declared:
        assert hasattr(lib, name)


def test_library_does_not_need_libcuda(lib):
    out = subprocess.run(["readelf", "-d", bw.library_path()], capture_output=True, text=True, check=True).stdout
    assert "libcuda.so" not in out  # driver calls go through the runtime's entry-point lookup


def test_library_is_built_for_sm100a():
    """The build compiles for sm_100a and nothing else (the kernels use
    tcgen05 and TMA; a device of another architecture is refused at run
    time with BONSAI_ERR_ARCH)."""
    cmd = bw_build.command()
    gencodes = [cmd[i + 1] for i, a in enumerate(cmd) if a == "-gencode"]
    assert gencodes == ["arch=compute_100a,code=sm_100a"]
    assert not any(a.startswith(("-arch", "--gpu-architecture")) for a in cmd)


def test_sizes(lib):
    assert bw.packed_bytes(3072, 9216, "ternary") == 3072 * 9216 // 4
    assert bw.packed_bytes(3072, 9216, "binary") == 3072 * 9216 // 8
    assert bw.scale_bytes(3072, 9216) == 3072 * 72 * 2
    assert bw.packed_bytes(8, 100, "ternary") == 0  # partial group
    assert bw.packed_bytes(3072, 9216, "ternary_b3") == 3072 * 112 * (9216 // 512)  # 112-byte blocks of 4 groups
    assert bw.packed_bytes(8, 640, "ternary_b3") == 8 * 112 * 2  # a partial last block still takes 112 bytes
    assert lib.bonsai_packed_bytes(8, 128, 4) == 0  # unknown mode
    assert lib.bonsai_packed_bytes(-1, 128, 2) == 0


def test_argument_errors_before_any_device_work(lib):
    P = None
    assert lib.bonsai_pack(P, 4, 128, 4, P, P) == 1  # mode
    assert lib.bonsai_pack(P, 4, 100, 2, P, P) == 2  # K % 128
    assert lib.bonsai_pack(P, -4, 128, 2, P, P) == 2
    assert lib.bonsai_pack(P, 0, 128, 2, P, P) == 0  # empty: no-op
    assert lib.bonsai_pack(P, 4, 128, 2, P, P) == 1  # null with data
    assert lib.bonsai_pack(8, 4, 128, 2, 16, P) == 3  # misaligned
    assert lib.bonsai_dequant(P, P, 4, 130, 1, P, P) == 2
    assert lib.bonsai_dequant(16, 16, 4, 128, 1, 24, P) == 3
    assert lib.bonsai_lowbit_gemm(P, P, P, 4, 4, 128, 0, P, P) == 1
    assert lib.bonsai_lowbit_gemm(P, P, P, 4, 4, 129, 2, P, P) == 2
    assert lib.bonsai_lowbit_gemm(P, P, P, 0, 4, 128, 2, P, P) == 0
    assert lib.bonsai_lowbit_gemm(P, P, P, 4, 4, 128, 2, P, P) == 1
    assert lib.bonsai_lowbit_gemm(P, P, P, 4, 4, 128, 2, 8, P) == 3
    assert lib.bonsai_lowbit_gemm(P, P, P, 1 << 31, 4, 128, 2, 16, P) == 2
    # 4-bit group-affine weights
    assert lib.bonsai_hqq4_packed_bytes(8, 256) == 8 * 256 // 2 and lib.bonsai_hqq4_packed_bytes(8, 100) == 0
    assert lib.bonsai_hqq4_pack(P, 4, 100, P, P) == 2
    assert lib.bonsai_hqq4_pack(P, 4, 128, P, P) == 1
    assert lib.bonsai_hqq4_dequant(16, 16, P, 4, 128, 16, P) == 1  # null zeros
    assert lib.bonsai_hqq4_gemm(P, P, P, P, 0, 4, 128, P, P) == 0
    assert lib.bonsai_hqq4_gemm(16, 16, 16, 24, 4, 4, 128, 16, P) == 3  # misaligned zeros
    # host-buffer form: A_host, packed, scales, M, N, K, mode, out_host, A_dev, out_dev, stream
    H = 16
    assert lib.bonsai_lowbit_gemm_host(H, H, H, 4, 4, 128, 0, H, H, H, P) == 1  # mode
    assert lib.bonsai_lowbit_gemm_host(H, H, H, 4, 4, 129, 2, H, H, H, P) == 2  # K % 128
    assert lib.bonsai_lowbit_gemm_host(P, P, P, 0, 4, 128, 2, P, P, P, P) == 0  # empty: no-op
    assert lib.bonsai_lowbit_gemm_host(P, H, H, 4, 4, 128, 2, H, H, H, P) == 1  # null host input
    assert lib.bonsai_lowbit_gemm_host(H, H, H, 4, 4, 128, 2, H, P, H, P) == 1  # null work buffer
    assert lib.bonsai_lowbit_gemm_host(H, H, H, 4, 4, 128, 2, H, 8, H, P) == 3  # misaligned work buffer


def test_batch_argument_errors_before_any_device_work(lib):
    Prob = bw.GemmProblem

    def call(problems, mode=2, count=None):
        arr = (Prob * max(len(problems), 1))(*problems)
        return lib.bonsai_lowbit_gemm_batch(arr, len(problems) if count is None else count, mode, None)

    ok = Prob(16, 16, 16, 16, 4, 8, 128)
    assert call([ok], mode=0) == 1  # mode
    assert call([ok], mode=4) == 1  # the 4-bit weights have no batch form
    assert call([ok], count=-1) == 1
    assert lib.bonsai_lowbit_gemm_batch(None, 2, 2, None) == 1  # no array
    assert lib.bonsai_lowbit_gemm_batch(None, 0, 2, None) == 0  # empty batch: no-op
    assert call([Prob(None, None, None, None, 0, 8, 128), Prob(None, None, None, None, 4, 0, 256)]) == 0  # empty
    assert call([ok, Prob(16, 16, 16, 16, 4, 8, 100)]) == 2  # K % 128 in the second problem
    assert call([ok, Prob(16, 16, 16, 16, -1, 8, 128)]) == 2
    assert call([Prob(16, 16, 16, 16, 1 << 31, 8, 128)]) == 2
    assert call([ok, Prob(16, None, 16, 16, 4, 8, 128)]) == 1  # null weights with data
    assert call([Prob(16, 16, 16, None, 4, 8, 128)]) == 1  # null out
    assert call([ok, Prob(16, 16, 24, 16, 4, 8, 128)]) == 3  # misaligned scales
    assert call([Prob(None, None, None, 8, 4, 8, 0)]) == 3  # K = 0 still writes out: aligned


def test_c_program_uses_the_abi(lib, tmp_path):
    """A C99 program built against include/bonsai.h and linked with
    libbonsai.so gets the documented sizes, status strings and argument
    errors (no device work, so it runs without a GPU)."""
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(bw.library_path())
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "abi_check.c"), "-L", libdir, "-lbonsai",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stderr


def test_status_strings(lib):
    for s in range(8):
        assert bw.status_string(s) != "unknown status"
    assert bw.status_string(99) == "unknown status"


def _imports(path):
    text = open(path, encoding="utf-8").read()
    return set(re.findall(r"^\s*(?:from|import)\s+([\w\.]+)", text, flags=re.M))


def _includes(path):
    return set(re.findall(r'#include\s+[<"]([^>"]+)[>"]', open(path, encoding="utf-8").read()))


def test_cuda_path_and_oracle_share_nothing():
    pkg = os.path.join(ROOT, "bit_weight_gemm_b200")
    orc = os.path.join(ROOT, "oracle")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            p = os.path.join(dirpath, f)
            if f.endswith(".py"):
                assert not any(i.split(".")[0] in ("oracle", "workloads") for i in _imports(p)), p
            if f.endswith((".cu", ".cuh", ".h")):
                assert not any("oracle" in i for i in _includes(p)), p
    for f in os.listdir(orc):
        p = os.path.join(orc, f)
        if f.endswith(".py"):
            assert not any(i.split(".")[0] in ("bit_weight_gemm_b200", "workloads") for i in _imports(p)), p
        if f.endswith(".c"):
            assert all(i in ("math.h", "pthread.h", "stdint.h", "stdlib.h", "string.h") for i in _includes(p)), p
