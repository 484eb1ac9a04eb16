"""Self-test of the sm_100a building blocks (tests/cuda/tc_selftest.cu): TMA
loads with the 128-byte swizzle, tcgen05.mma with shared-memory K-major
operands and with A from tensor memory against an MN-major B, and the bounded
mbarrier wait giving up with MONARCH_ERR_TIMEOUT instead of hanging."""
import ctypes
import os
import subprocess

import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cuda", "tc_selftest.cu")
LIB = os.path.join(HERE, "_build", "libtcselftest.so")
DEPS = [SRC, os.path.join(HERE, "..", "structured_attention_video_b200", "csrc",
                          "tc_primitives.cuh")]


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB) or any(os.path.getmtime(d) > os.path.getmtime(LIB) for d in DEPS):
        os.makedirs(os.path.dirname(LIB), exist_ok=True)
        nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
        subprocess.run([nvcc, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-Xcompiler", "-fPIC", "-shared", SRC, "-o", LIB], check=True)
    so = ctypes.CDLL(LIB)
    vp = ctypes.c_void_p
    so.selftest_gemm.argtypes = [vp, vp, ctypes.c_int, vp, vp, vp]
    so.selftest_wait.argtypes = [vp, ctypes.c_longlong, vp]
    so.selftest_exp2.argtypes = [vp, vp, vp, ctypes.c_int]
    return so


@pytest.mark.parametrize("n", [64, 80, 128])
def test_ss_and_ts_mma(lib, n):
    g = torch.Generator().manual_seed(n)
    a = torch.randn(128, 128, generator=g).to(torch.bfloat16).cuda()
    b = torch.randn(n, 128, generator=g).to(torch.bfloat16).cuda()
    d = torch.zeros(128, n, device="cuda")
    e = torch.zeros(128, 128, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.selftest_gemm(a.data_ptr(), b.data_ptr(), n, d.data_ptr(), e.data_ptr(),
                             st.data_ptr()) == 0
    assert int(st.item()) == 0
    d_ref = a.double() @ b.double().T
    assert ((d.double() - d_ref).norm() / d_ref.norm()).item() < 1e-5
    e_ref = d.to(torch.bfloat16).double() @ b.double()
    assert ((e.double() - e_ref).norm() / e_ref.norm()).item() < 1e-5


def test_bounded_wait_gives_up(lib):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    assert lib.selftest_wait(st.data_ptr(), 4096, res.data_ptr()) == 0
    assert int(res.item()) == 0          # the wait returned "not completed"
    assert int(st.item()) == 7           # MONARCH_ERR_TIMEOUT recorded
    assert torch.ones(4, device="cuda").sum().item() == 4   # the context is still usable


def test_polynomial_exp2_within_its_error_bound(lib):
    """exp2_poly_x2 (Cody-Waite reduction, degree-3 minimax on [0, 1)) against 2^d in
    float64: relative error <= 1e-4 (the fit's 7.5e-5 plus float32 rounding) down to
    2^-125; below that a non-negative value of at most 2^-125 (at 2^-126 the result's
    exponent field reaches zero and precision drops); and it agrees
    with the MUFU exponential it replaces to the same bound."""
    d = torch.cat([torch.linspace(-130.0, 0.0, 200001, dtype=torch.float64),
                   torch.tensor([0.0, -1e-7, -0.5, -1.0, -126.0, -126.5, -127.0, -1e4,
                                 -3e38], dtype=torch.float64)]).float()
    n = d.numel()
    x = d.cuda()
    poly = torch.empty(n, device="cuda")
    mufu = torch.empty(n, device="cuda")
    assert lib.selftest_exp2(x.data_ptr(), poly.data_ptr(), mufu.data_ptr(), n) == 0
    ref = torch.exp2(d.double())
    got = poly.cpu().double()
    normal = ref >= 2.0 ** -125
    rel = ((got[normal] - ref[normal]).abs() / ref[normal]).max().item()
    assert rel <= 1e-4
    assert bool((got[~normal] >= 0).all()) and bool((got[~normal] <= 2.0 ** -125).all())
    m = mufu.cpu().double()
    assert ((got[normal] - m[normal]).abs() / m[normal]).max().item() <= 1.2e-4
