"""GPU tests of the user-level calls: isa_attention (device tensors, pinned
host tensors, with the decoupled RoPE), the head-sharded helper's CUDA path
and CUDA-graph capture of plan + forward + backward.  Each must give exactly
the bits of the explicit calls (every head is computed independently, so
slicing heads changes nothing)."""
import numpy as np
import pytest
import torch

from parity import to_torch_bf16
from workloads import Workload, generate_bits, generate_dout_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_attention_coarse_b200 import build
    build.build()
    import block_sparse_attention_coarse_b200 as I
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return I


@pytest.fixture(scope="module")
def case(isa):
    w = Workload("api", 2, 3, 128, 700, 333, block=64, alpha_s=0.25, alpha_f=0.5, alpha_ns=0.125, seed=95)
    qb, kb, vb = generate_bits(w)
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block, w.alpha_s, w.alpha_f, w.alpha_ns)
    return w, p, qb, kb, vb


def test_isa_attention_device_and_pinned_host(isa, case):
    w, p, qb, kb, vb = case
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    ws = isa.plan(q, k, v, p)
    ref = isa.forward(q, k, v, ws, p)
    dev = isa.isa_attention(q, k, v, p)
    host_in = [to_torch_bf16(x, device="cpu").pin_memory() for x in (qb, kb, vb)]
    host = isa.isa_attention(*host_in, p)
    torch.cuda.synchronize()
    assert not host.is_cuda
    assert torch.equal(dev, ref)
    assert torch.equal(host, ref.cpu())


def test_isa_attention_with_rope(isa, case):
    w, p, qb, kb, vb = case
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    qr, kr = isa.rope(q, k, p, 10000.0)
    ref = isa.forward(qr, kr, v, isa.plan(qr, kr, v, p), p)
    got = isa.isa_attention(q, k, v, p, rope_base=10000.0)
    host = isa.isa_attention(*(to_torch_bf16(x, device="cpu").pin_memory() for x in (qb, kb, vb)), p,
                             rope_base=10000.0)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    assert torch.equal(host, ref.cpu())


@pytest.mark.parametrize("world", [2, 4])
def test_head_sharded_cuda_path_equals_full_run(isa, case, world):
    from block_sparse_attention_coarse_b200 import shard
    w, p, qb, kb, vb = case
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    full = isa.isa_attention(q, k, v, p).reshape(w.BH, w.L, w.D)
    parts = []
    for r in range(world):
        out, (lo, hi) = shard.isa_attention_heads(q, k, v, p, r, world)
        assert (lo, hi) == shard.head_range(w.BH, r, world)
        parts.append(out)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=0), full)


def test_cuda_graph_capture_and_replay(isa, case):
    """plan + forward + backward are stream-ordered and allocate nothing, so
    they capture into one CUDA graph; replays on new inputs give exactly
    the eager results."""
    w, p, qb, kb, vb = case
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    do = to_torch_bf16(generate_dout_bits(w))
    ws = isa.alloc_workspace(p, q.device)
    lse = torch.empty(w.B, w.H, w.L, dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    bws = torch.empty(isa.backward_workspace_size(p), dtype=torch.uint8, device="cuda")
    qs, ks, vs, dos = (t.clone() for t in (q, k, v, do))   # static inputs of the graph

    def step():
        isa.plan(qs, ks, vs, p, ws)
        isa.forward(qs, ks, vs, ws, p, out=out, lse=lse)
        isa.backward(qs, ks, vs, ws, p, out, lse, dos, dq, dk, dv, bws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()   # warm-up on the capture stream (library initialisation, kernel attributes)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for scale in (1.0, 0.5):
        for s, t in ((qs, q), (ks, k), (vs, v), (dos, do)):
            s.copy_(t * scale)
        graph.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (out, dq, dk, dv)]
        step()
        torch.cuda.synchronize()
        for a, b in zip(got, (out, dq, dk, dv)):
            assert torch.equal(a, b)
    assert int(isa.plan_view(p, ws)["status"].item()) == 0
