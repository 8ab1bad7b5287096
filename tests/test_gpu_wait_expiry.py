"""Failure detection without a GPU fault: the tensor-core kernels' bounded wait, made to run out.

A one-CTA self-test kernel holds tensor memory and waits, with the kernels' own wait routine, on an
mbarrier that nothing arrives at, under a 1 ms limit.  The wait must give up, set bit 0 of the
status word at the start of a libgdn workspace, raise the CTA's abort flag for every thread, and
the kernel must release its tensor memory and return; gdn_workspace_status then reports
GDN_ERR_TIMEOUT.  The control case arrives at the barrier and must report success.  Afterwards the
library's kernels still run on the same context.
"""
import ctypes
import time

import pytest
import torch

from gated_delta_rule_76_b200 import build as gbuild
from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import draw

pytestmark = pytest.mark.gpu

GDN_OK, GDN_ERR_TIMEOUT = 0, 5


@pytest.fixture(scope="module")
def selftest():
    gbuild.build()
    L = ctypes.CDLL(gbuild.SELFTEST_LIB)
    L.gdn_selftest_wait_expiry.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_int,
                                           ctypes.c_void_p]
    L.gdn_selftest_wait_expiry.restype = ctypes.c_int
    return L


def run(selftest, limit_ns, arrive):
    lib = gdn.load()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")  # a workspace: status word at offset 0
    out = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    rc = selftest.gdn_selftest_wait_expiry(ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                           limit_ns, arrive, None)
    assert rc == 0
    status = lib.gdn_workspace_status(ctypes.c_void_p(ws.data_ptr()), None)
    elapsed = time.perf_counter() - t0
    return status, out.cpu().tolist(), elapsed, lib


def test_expired_wait_sets_the_status_word_and_returns(selftest):
    limit_ns = 1_000_000  # 1 ms
    status, out, elapsed, lib = run(selftest, limit_ns, arrive=0)
    assert status == GDN_ERR_TIMEOUT, lib.gdn_last_error().decode()
    assert "bounded wait" in lib.gdn_last_error().decode()
    assert out[0] == 0, "the wait must report failure"
    assert out[1] == 128, "every thread of the CTA must see the abort flag"
    assert elapsed < 5.0, "the kernel must return soon after the limit"


def test_wait_that_completes_reports_success(selftest):
    status, out, _, _ = run(selftest, 1_000_000_000, arrive=1)
    assert status == GDN_OK
    assert out == [1, 0]


def test_library_runs_after_an_expired_wait(selftest):
    run(selftest, 1_000_000, arrive=0)
    x = draw(1, 130, 2, 2, 128, 128, alpha_per_channel=True, gates_per_channel=True, dtype="bf16",
             gate_dtype="bf16", seed=41, has_h0=True)
    g = {k: v.cuda() for k, v in x.items()}
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], h0=g["h0"])
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(ht).all()
