"""GPU parity at the largest plan the library accepts: 8192 blocks per head
and 6144 kept blocks per head (131072 + 131072 tokens in blocks of 32, with
alpha_s = 0.5 keeping half of the 4096 context blocks).  Every planning
kernel then runs at its largest shared-memory footprint (the exact-list
kernel holds 8 rows of 6144 scores), and the attention kernel walks 1536 KV
tiles per sharp item and 384 exact plus 48 pooled tiles per flat item.
The plan is compared with the oracle under the margin rules, and the
outputs of a seeded sample of query blocks element by element (against the
oracle run on the GPU's plan where the two plans differ inside the margin)."""
import pytest
import torch

from parity import check_case
from workloads import Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_attention_coarse_b200 import build
    build.build()
    import block_sparse_attention_coarse_b200 as I
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return I


def test_forward_at_the_block_limits(isa):
    w = Workload("max_blocks", 1, 1, 128, 131072, 131072, block=32, alpha_s=0.5, seed=5000)
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block, w.alpha_s, w.alpha_f, w.alpha_ns)
    v = isa.plan_view(p, torch.empty(isa.workspace_size(p), dtype=torch.uint8, device="cuda"))
    assert (v["T"], v["T_kv"], v["n_flat"], v["n_exact"]) == (8192, 6144, 4096, 384)
    # With 6144 kept blocks the 384th and 385th scores of a row are often
    # closer than fp32 can order, so a sampled flat block may take another
    # (within-margin) exact list than the oracle's; its output is then
    # compared with the oracle run on the GPU's own (validated) list.
    check_case(isa, w, heads=[0], blocks_per_head=8)
