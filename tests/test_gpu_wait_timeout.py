"""Failure detection without a GPU fault: a kernel whose bounded wait can never be satisfied gives up
after its limit, raises the workspace status word and returns; the host reads SV_ERR_TIMEOUT and the
CUDA context stays usable for ordinary calls afterwards."""

import time

import numpy as np
import pytest
import torch

import oracle
from block_causal_linear_relu_b200.inputs import draw_qkv, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from block_causal_linear_relu_b200 import build
    build.build()
    import block_causal_linear_relu_b200 as m
    m.load()
    return m


def test_bounded_wait_expires_and_context_survives(sv):
    ws = sv.Workspace(4096, torch.device("cuda:0"))
    assert ws.status() == 0
    t0 = time.perf_counter()
    sv.sv_selftest_wait_timeout(ws)
    code = ws.status()                          # synchronises: returns once the waiters gave up
    waited = time.perf_counter() - t0
    assert code & 0x80000000, hex(code)         # the timeout bit
    assert code & 0xFF00 == 0x7E00, hex(code)   # raised by the self-test's waiters
    assert 1.0 < waited < 60.0
    assert ws.status() == 0                     # reading the word cleared it

    # the context still runs ordinary work, and correctly
    q, k, v = draw_qkv((1, 2, 300, 64), 11, "bf16")
    dq, dk, dv = (torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
                  for x in (q, k, v))
    o = sv.sv_block_causal_attn(dq, dk, dv, 128, eps=1e-6)
    torch.cuda.synchronize()
    want = oracle.block_causal_attn(*(to_f64(x, "bf16") for x in (q, k, v)), 128, 1e-6)[0]
    assert oracle.max_rel_err(o.float().cpu().numpy().astype(np.float64), want) < 2e-2


def test_selftest_refuses_bad_workspace(sv):
    import ctypes
    ws = sv.Workspace(4096, torch.device("cuda:0"))
    lib = sv.load()
    invalid = 1  # SV_ERR_INVALID_ARG
    assert lib.sv_selftest_wait_timeout(None, 4096, None) == invalid
    assert lib.sv_selftest_wait_timeout(ctypes.c_void_p(ws.view.data_ptr() + 8), 4088, None) == invalid
    assert lib.sv_selftest_wait_timeout(ws.ptr, 64, None) == invalid
    assert ws.status() == 0                     # nothing was launched


def test_binding_raises_on_the_next_call_after_a_timeout(sv):
    # a kernel that gives up a bounded wait also writes its code into the workspace's host-mapped
    # mirror word; the binding reads that word before each call and raises instead of launching on a
    # workspace whose last call did not complete (no per-call synchronisation)
    st = draw_qkv((1, 2, 300, 64), 12, "bf16")
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda() for x in st)
    ws = sv.make_workspace(sv.SV_OP_LINATTN_FWD, q)
    sv.sv_selftest_wait_timeout(ws)
    torch.cuda.synchronize()                    # the waiters give up after about 2 s
    with pytest.raises(sv.SvError) as err:
        sv.sv_linattn_fwd(q, k, v, eps=1e-6, ws=ws)
    assert err.value.status == 4                # SV_ERR_TIMEOUT
    # the check read and cleared the word: the next call runs, and correctly
    o = sv.sv_linattn_fwd(q, k, v, eps=1e-6, ws=ws)
    torch.cuda.synchronize()
    want = oracle.linattn_fwd(*(to_f64(x, "bf16") for x in st), 1e-6)
    assert oracle.max_rel_err(o.float().cpu().numpy().astype(np.float64), want) < 2e-2
    ws.check()                                  # nothing reported since


def test_mirror_needs_host_memory_the_device_can_write(sv):
    import ctypes
    lib = sv.load()
    ws = sv.Workspace(4096, torch.device("cuda:0"))
    dev_word = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.sv_workspace_set_mirror(ws.ptr, ws.nbytes, ctypes.c_void_p(dev_word.data_ptr()), None) == 1
    assert b"page-locked" in lib.sv_last_error()
    assert lib.sv_workspace_set_mirror(ws.ptr, ws.nbytes, None, None) == 0   # removing it is allowed
