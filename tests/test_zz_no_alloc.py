"""isa_forward_static: the forward pass for callers that cannot allocate.

Code that must not call cudaMalloc -- an allocator or memory-pool callback, a
real-time loop that forbids allocation, a binding without a device allocator
-- cannot hand the library a plan workspace.  isa_forward_static keeps the
plan in a fixed 16 MiB device array inside the library instead.  These tests
call it through the C interface and check that its output matches the
regular isa_plan + isa_forward path (the caller-allocated workspace) within
the tolerance of the other GPU tests, and indeed bit for bit (the same
kernels on the same inputs), on consecutive calls that reuse the shared
array; that its status word reports a device wait that ran out; and that a
problem too large for the array is refused with a clear error before
anything runs.  Collected last so that a run stopping at
its first failure has already run every other test; it also passes alone.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity import OUT_MAX_ABS, OUT_MEAN_ABS, to_torch_bf16
from workloads import Workload, generate_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_attention_coarse_b200 import build
    build.build()
    import block_sparse_attention_coarse_b200 as I
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return I


def inputs(isa, w):
    q, k, v = (to_torch_bf16(x) for x in generate_bits(w))
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block, w.alpha_s, w.alpha_f, w.alpha_ns)
    return q, k, v, p


def static_forward(isa, q, k, v, p):
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:-1], float("nan"), dtype=torch.float32, device=q.device)
    st = isa.load_library().isa_forward_static(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                               out.data_ptr(), lse.data_ptr(),
                                               torch.cuda.current_stream().cuda_stream)
    assert st == isa.ISA_OK, isa.load_library().isa_last_error()
    return out, lse


def close(a, b):
    d = (a.float() - b.float()).abs()
    return float(d.max()) <= OUT_MAX_ABS and float(d.mean()) <= OUT_MEAN_ABS


def static_status(isa):
    """The status word of the fixed array on the current device (a copy into
    a host int32 through isa_forward_static_status)."""
    word = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st = isa.load_library().isa_forward_static_status(torch.cuda.current_device(), word.data_ptr(),
                                                      torch.cuda.current_stream().cuda_stream)
    assert st == isa.ISA_OK, isa.load_library().isa_last_error()
    return int(word.item())


def test_static_scratch_matches_workspace_path_on_consecutive_calls(isa):
    w = Workload("noalloc", 1, 4, 128, 700, 450, block=64, alpha_s=0.25, alpha_f=0.5, alpha_ns=0.2, seed=91)
    q, k, v, p = inputs(isa, w)
    assert isa.workspace_size(p) <= 16 << 20
    lse_ref = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    ref = isa.forward(q, k, v, isa.plan(q, k, v, p), p, lse=lse_ref)
    for _ in range(2):
        out, lse = static_forward(isa, q, k, v, p)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert close(out, ref)
        # the same kernels on the same inputs: bit for bit the same results,
        # which a stale plan entry left in the shared array would break
        assert torch.equal(out, ref) and torch.equal(lse, lse_ref)
        assert static_status(isa) == isa.ISA_OK
    # a different problem on the next call: the shared array is rewritten
    w2 = Workload("noalloc2", 2, 2, 64, 333, 97, block=32, alpha_s=0.3, alpha_f=0.5, alpha_ns=0.2, seed=92)
    q2, k2, v2, p2 = inputs(isa, w2)
    ref2 = isa.forward(q2, k2, v2, isa.plan(q2, k2, v2, p2), p2)
    out2, _ = static_forward(isa, q2, k2, v2, p2)
    torch.cuda.synchronize()
    assert close(out2, ref2) and torch.equal(out2, ref2)


def test_static_status_reports_a_device_timeout(isa):
    """A device wait that runs out inside isa_forward_static (fault injection
    makes the attention kernel wait on a barrier nothing arrives on) is
    visible through isa_forward_static_status; the next call clears it and
    is correct again."""
    w = Workload("noalloc_to", 1, 2, 64, 256, 128, block=64, alpha_s=0.5, alpha_f=0.5, alpha_ns=0.25, seed=93)
    q, k, v, p = inputs(isa, w)
    ref = isa.forward(q, k, v, isa.plan(q, k, v, p), p)
    isa.set_wait_timeout_ns(2_000_000)
    isa.set_fault_injection(1)
    try:
        static_forward(isa, q, k, v, p)
        torch.cuda.synchronize()
    finally:
        isa.set_fault_injection(0)
        isa.set_wait_timeout_ns(0)
    assert static_status(isa) == isa.ISA_ERR_DEVICE_TIMEOUT
    out, _ = static_forward(isa, q, k, v, p)
    torch.cuda.synchronize()
    assert static_status(isa) == isa.ISA_OK
    assert torch.equal(out, ref)


def test_static_scratch_refuses_problems_larger_than_the_array(isa):
    lib = isa.load_library()
    p = isa.make_params(2, 40, 128, 16384, 16384)          # plan needs about 81 MB
    assert isa.workspace_size(p) > 16 << 20
    st = lib.isa_forward_static(ctypes.byref(p), 1 << 20, 1 << 20, 1 << 20, 1 << 20, None, None)
    assert st == isa.ISA_ERR_WORKSPACE
    assert b"fixed device array" in lib.isa_last_error()
