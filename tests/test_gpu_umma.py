"""The sm_100a building blocks of the tensor-core kernels, checked in isolation on the GPU:
tcgen05 MMA with both operands in 128-byte-swizzled shared memory, accumulation into tensor
memory, A taken from tensor memory, and a 4-D TMA box with the 128-byte swizzle (including the
zero fill past the end of a sequence)."""
import ctypes

import pytest
import torch

from gated_delta_rule_76_b200 import build as gbuild

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    L = ctypes.CDLL(gbuild.SELFTEST_LIB)
    P = ctypes.c_void_p
    L.gdn_selftest_mma.argtypes = [P] * 9
    L.gdn_selftest_mma.restype = ctypes.c_int
    L.gdn_selftest_mma_mn.argtypes = [P] * 8
    L.gdn_selftest_mma_mn.restype = ctypes.c_int
    L.gdn_selftest_tma.argtypes = [P] + [ctypes.c_int] * 7 + [P, P, P]
    L.gdn_selftest_tma.restype = ctypes.c_int
    return L


def p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_tcgen05_mma_shared_and_tensor_memory_operands(lib):
    g = torch.Generator().manual_seed(0)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    A, B1, A2, B3, B2 = mk(128, 128), mk(64, 128), mk(128, 64), mk(64, 64), mk(128, 128)
    dev = [t.cuda() for t in (A, B1, A2, B3, B2)]
    D1 = torch.full((128, 64), float("nan"), device="cuda")
    D2 = torch.full((128, 128), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.gdn_selftest_mma(*[p(t) for t in dev], p(D1), p(D2), p(err),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0 and int(err.item()) == 0
    ref1 = A.double() @ B1.double().T + A2.double() @ B3.double().T
    ref2 = A.double() @ B2.double().T
    for got, ref, name in ((D1, ref1, "ss + accumulate"), (D2, ref2, "A from tensor memory")):
        e = (got.cpu().double() - ref).abs().max() / ref.abs().max()
        assert e < 1e-5, f"{name}: relative error {e:.2e}"


def test_tcgen05_mma_mn_major_operands(lib):
    g = torch.Generator().manual_seed(2)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    Ak, X, B2 = mk(128, 64), mk(64, 128), mk(64, 64)
    dev = [t.cuda() for t in (Ak, X, B2)]
    D1 = torch.full((128, 128), float("nan"), device="cuda")
    D2 = torch.full((128, 64), float("nan"), device="cuda")
    D3 = torch.full((128, 128), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.gdn_selftest_mma_mn(*[p(t) for t in dev], p(D1), p(D2), p(D3), p(err),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0 and int(err.item()) == 0
    ref1 = Ak.double() @ X.double()
    ref2 = X.double().T @ B2.double().T
    for got, ref, name in ((D1, ref1, "B MN-major"), (D2, ref2, "A MN-major, 128-row tile"),
                           (D3, ref1, "A in tensor memory, B MN-major")):
        e = (got.cpu().double() - ref).abs().max() / ref.abs().max()
        assert e < 1e-5, f"{name}: relative error {e:.2e}"


@pytest.mark.parametrize("c0,hh,t0,bb", [(0, 0, 0, 0), (64, 2, 64, 1)])
def test_tma_box_with_128b_swizzle(lib, c0, hh, t0, bb):
    B, T, H = 2, 100, 3
    x = torch.randn(B, T, H, 128, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).cuda()
    out = torch.full((64, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.gdn_selftest_tma(p(x), B, T, H, c0, hh, t0, bb, p(out), p(err),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0 and int(err.item()) == 0
    ref = torch.zeros(64, 64, dtype=torch.bfloat16)
    n = min(64, T - t0)
    ref[:n] = x[bb, t0:t0 + n, hh, c0:c0 + 64].cpu()
    assert torch.equal(out.cpu(), ref)
