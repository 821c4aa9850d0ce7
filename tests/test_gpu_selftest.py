"""tcgen05 / TMA layout self-checks on the GPU: one-CTA products through the test-only libfa_selftest.so, using
the operand forms the attention kernels rely on, compared with a float32 product of the same 16-bit values."""
import ctypes
import os

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SELFTEST = os.path.join(ROOT, "exact_io_aware_76_b200", "libfa_selftest.so")

VARIANTS = {0: "A K-major smem, B K-major smem", 1: "A K-major smem, B MN-major smem",
            2: "A TMEM, B MN-major smem", 3: "A MN-major smem, B MN-major smem"}


@pytest.fixture(scope="module")
def st():
    L = ctypes.CDLL(SELFTEST)
    L.fa_selftest_umma.restype = ctypes.c_int
    L.fa_selftest_umma.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int]
    return L


@pytest.mark.gpu
@pytest.mark.parametrize("variant", sorted(VARIANTS))
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("K", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_umma_layouts(st, variant, N, K, dtype):
    g = torch.Generator(device="cuda")
    g.manual_seed(7 + variant * 100 + N + K)
    if variant == 3:
        a = torch.randn(K, 128, device="cuda", generator=g).to(dtype)  # stored [K][M]
        a_mk = a.float().t()
    else:
        a = torch.randn(128, K, device="cuda", generator=g).to(dtype)
        a_mk = a.float()
    if variant == 0:
        b = torch.randn(N, K, device="cuda", generator=g).to(dtype)  # stored [N][K]
        b_kn = b.float().t()
    else:
        b = torch.randn(K, N, device="cuda", generator=g).to(dtype)  # stored [K][N]
        b_kn = b.float()
    c = torch.full((128, N), float("nan"), device="cuda", dtype=torch.float32)
    rc = st.fa_selftest_umma(variant, a.data_ptr(), b.data_ptr(), c.data_ptr(), N, K, int(dtype == torch.bfloat16))
    assert rc == 0, rc
    ref = a_mk.double() @ b_kn.double()
    err = (c.double() - ref).abs().max().item()
    assert err <= 1e-3 * max(1.0, ref.abs().max().item()), (VARIANTS[variant], err)


@pytest.mark.gpu
def test_bounded_wait_gives_up_and_reports_timeout(st):
    """A wait that nothing satisfies (an mbarrier no thread arrives on) must give up after its limit, record
    FA_ERR_TIMEOUT in the device status word and return; the context stays usable afterwards."""
    import time

    import exact_io_aware_76_b200 as fa

    st.fa_selftest_wait_timeout.restype = ctypes.c_int
    st.fa_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_int)]
    waited_ok = ctypes.c_int(-1)
    t0 = time.perf_counter()
    status = st.fa_selftest_wait_timeout(10_000_000, ctypes.byref(waited_ok))  # 10 ms limit
    elapsed = time.perf_counter() - t0
    assert status == -4, status
    assert waited_ok.value == 0
    assert elapsed < 5.0
    # The GPU still works: a normal forward runs and the product library's status word is clean.
    q = torch.randn(1, 128, 1, 64, device="cuda").half()
    out, lse = fa.fwd(q, q, q)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and fa.device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("variant,N", [(0, 64), (0, 128), (1, 128)])
def test_e4m3_layouts(st, variant, N):
    """8-bit (e4m3) tcgen05 products: the S = Q K^T form from shared memory, and the O = P V form with A in TMEM
    (four consecutive K elements per 32-bit column) and an MN-major B."""
    st.fa_selftest_f8.restype = ctypes.c_int
    st.fa_selftest_f8.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    g = torch.Generator(device="cuda")
    g.manual_seed(77 + variant + N)
    a = (torch.randn(128, 128, device="cuda", generator=g) * 2).to(torch.float8_e4m3fn)
    b = (torch.randn(N, 128, device="cuda", generator=g) * 2).to(torch.float8_e4m3fn) if variant == 0 else \
        (torch.randn(128, N, device="cuda", generator=g) * 2).to(torch.float8_e4m3fn)
    c = torch.full((128, N), float("nan"), device="cuda", dtype=torch.float32)
    rc = st.fa_selftest_f8(variant, a.view(torch.uint8).data_ptr(), b.view(torch.uint8).data_ptr(), c.data_ptr(), N)
    assert rc == 0, rc
    ref = a.double() @ (b.double().t() if variant == 0 else b.double())
    err = (c.double() - ref).abs().max().item()
    assert err <= 1e-3 * max(1.0, ref.abs().max().item()), err


@pytest.mark.gpu
def test_exp2_on_the_fma_pipe(st):
    """The forward softmax computes some exponentials as exp2_poly2 (range reduction to the nearest integer
    plus a degree-3 polynomial). Against fp64 exp2: relative error <= 1e-4 for x in [-125, 9] (the polynomial's
    fitted bound is 8.4e-5, plus fp32 evaluation), about ex2.approx's own accuracy order; x below -125 returns at
    most 2^-124 (a clamped, negligible weight); integers give exact powers of two up to the polynomial error."""
    import numpy as np

    st.fa_selftest_exp2.restype = ctypes.c_int
    st.fa_selftest_exp2.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    x = torch.cat([torch.linspace(-125.0, 9.0, 1 << 20, device="cuda"),
                   torch.rand(1 << 18, generator=g, device="cuda") * 134.0 - 125.0,
                   torch.arange(-125, 10, device="cuda", dtype=torch.float32),
                   torch.tensor([-0.5, 0.5, -0.49999997, 0.49999997, 0.0, -1e-30, 8.5], device="cuda"),
                   torch.tensor([-126.0, -200.0, -1e30, -3e38], device="cuda")])
    if x.numel() % 2:
        x = torch.cat([x, torch.zeros(1, device="cuda")])
    y = torch.empty_like(x)
    z = torch.empty_like(x)
    assert st.fa_selftest_exp2(x.data_ptr(), y.data_ptr(), z.data_ptr(), x.numel()) == 0
    xs = x.cpu().double().numpy()
    ys = y.cpu().double().numpy()
    zs = z.cpu().double().numpy()
    inside = xs >= -125.0
    ref = np.exp2(xs[inside])
    rel = np.abs(ys[inside] / ref - 1.0)
    rel_mufu = np.abs(zs[inside] / ref - 1.0)
    print("poly max rel %.3e, ex2.approx max rel %.3e" % (rel.max(), rel_mufu.max()))
    assert rel.max() <= 1e-4
    assert np.all((ys[~inside] > 0) & (ys[~inside] <= 2.0 ** -124))
