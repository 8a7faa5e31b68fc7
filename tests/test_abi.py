"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/isa.h declares, validates arguments on the host and sizes the
plan exactly as the oracle's counting rules say."""
import ctypes
import os
import re

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def isa():
    from block_sparse_attention_coarse_b200 import build
    build.build()
    import block_sparse_attention_coarse_b200 as I
    I.load_library()
    return I


def declared_functions():
    text = open(os.path.join(ROOT, "include", "isa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:isa_status|const char\*)\s+(isa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("isa_plan", "isa_forward", "isa_dense", "isa_plan_workspace_size", "isa_plan_view_get",
                     "isa_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(isa):
    lib = isa.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(isa.EXPORTS)
    assert "sm_100a" in isa.version()


@pytest.mark.parametrize("bad,status", [
    (dict(D=96), 2), (dict(block=16), 2), (dict(alpha_s=0.0), 1), (dict(alpha_s=1.5), 1), (dict(alpha_f=-0.1), 1),
    (dict(alpha_ns=1.01), 1), (dict(L_src=0), 1), (dict(L_ctx=-3), 1), (dict(B=0), 1),
    (dict(scale=float("nan")), 1), (dict(H=100000, L_src=400000, L_ctx=400000), 2),
])
def test_invalid_params_rejected_on_host(isa, bad, status):
    kw = dict(B=1, H=2, D=64, L_src=100, L_ctx=50, block=64, alpha_s=0.125, alpha_f=0.5, alpha_ns=0.0625)
    kw.update(bad)
    p = isa.make_params(**kw)
    with pytest.raises(isa.IsaError) as e:
        isa.workspace_size(p)
    assert e.value.status == status
    assert len(isa.load_library().isa_last_error()) > 0


def test_binding_defaults_match_the_oracle(isa):
    b = isa.make_params(1, 1, 64, 1, 1)
    o = O.Params(D=64, L_src=1, L_ctx=1)
    assert (b.alpha_s, b.alpha_f, b.alpha_ns, b.block) == (o.alpha_s, o.alpha_f, o.alpha_ns, o.block)
    assert b.scale == 0.0 and o.scale is None       # both select 1/sqrt(D)


def test_block_limits(isa):
    """8192 blocks and 6144 kept blocks per head are the largest plan
    accepted; one block more of either is refused before anything runs."""
    ok = isa.make_params(1, 1, 128, 131072, 131072, 32, 0.5)
    v, _ = fake_view(isa, ok)
    assert (v.T, v.T_kv) == (8192, 6144)
    for bad in (isa.make_params(1, 1, 128, 131072, 131073, 32, 0.25),            # T = 8193
                isa.make_params(1, 1, 128, 131072, 131072, 32, 2049 / 4096)):   # T_kv = 6145
        with pytest.raises(isa.IsaError) as e:
            isa.workspace_size(bad)
        assert e.value.status == 2 and "at most" in str(e.value)


def fake_view(isa, p):
    """Sizes from isa_plan_view_get; the workspace is never dereferenced."""
    lib = isa.load_library()
    n = isa.workspace_size(p)
    v = isa._PlanView()
    st = lib.isa_plan_view_get(ctypes.byref(p), ctypes.c_void_p(1 << 20), n, ctypes.byref(v))
    assert st == 0
    return v, n


@pytest.mark.parametrize("L_src,L_ctx,b,a_s,a_f,a_ns", [
    (1024, 1024, 64, 0.125, 0.5, 0.0625), (11884, 11884, 64, 0.125, 0.5, 0.0625),
    (16384, 16384, 64, 0.125, 0.5, 0.0625), (32768, 32768, 32, 0.125, 0.5, 0.0625),
    (100, 37, 32, 0.3, 0.7, 0.2), (5, 3, 64, 1.0, 0.0, 1.0), (65536, 65536, 64, 0.0625, 0.5, 0.03125),
    (300, 1, 32, 0.01, 1.0, 0.0),
])
def test_plan_counts_follow_the_oracle_rules(isa, L_src, L_ctx, b, a_s, a_f, a_ns):
    p = isa.make_params(1, 3, 128, L_src, L_ctx, b, a_s, a_f, a_ns)
    v, n = fake_view(isa, p)
    _, _, T_src, T_ctx = O.segment_blocks(L_src, L_ctx, b)
    T = T_src + T_ctx
    assert (v.T_src, v.T_ctx, v.T) == (T_src, T_ctx, T)
    assert v.K_sel == O.n_select(a_s, T_ctx)
    assert v.T_kv == T_src + v.K_sel
    assert v.n_flat == O.n_flat_blocks(a_f, T) and v.n_sharp == T - v.n_flat
    assert v.n_exact == O.n_exact_blocks(a_ns, v.T_kv)
    assert v.T_kv_pad % 128 == 0 and v.T_kv_pad >= v.T_kv
    assert v.bitmap_words == (v.T_kv + 31) // 32
    # every array lies inside the workspace, 256-byte aligned
    base = 1 << 20
    for name in ("Qc", "Kc", "Vc", "imp", "ctx_sel", "kept", "energy", "sharp_ids", "flat_ids", "exact",
                 "exact_bits", "Kp", "Vp", "status"):
        ptr = getattr(v, name)
        assert base <= ptr < base + n and (ptr - base) % 256 == 0, name


def test_workspace_too_small_is_rejected(isa):
    p = isa.make_params(1, 2, 64, 256, 256)
    n = isa.workspace_size(p)
    v = isa._PlanView()
    st = isa.load_library().isa_plan_view_get(ctypes.byref(p), ctypes.c_void_p(1 << 20), n - 1, ctypes.byref(v))
    assert st == 3


def test_null_and_misaligned_pointers_rejected_before_launch(isa):
    lib = isa.load_library()
    p = isa.make_params(1, 2, 64, 256, 256)
    n = isa.workspace_size(p)
    st = lib.isa_plan(ctypes.byref(p), None, 1 << 20, 1 << 20, 1 << 20, n, None)
    assert st == 1 and b"q is NULL" in lib.isa_last_error()
    st = lib.isa_forward(ctypes.byref(p), 1 << 20, (1 << 20) + 2, 1 << 20, 1 << 20, n, 1 << 20, None, None)
    assert st == 1 and b"aligned" in lib.isa_last_error()
    st = lib.isa_dense(ctypes.byref(p), 1 << 20, 1 << 20, 1 << 20, None, None, None, None)
    assert st == 1


def test_rope_arguments_rejected_before_launch(isa):
    """isa_rope checks the base, the pointers and the table size on the host
    (fake device addresses: nothing may be launched)."""
    lib = isa.load_library()
    p = isa.make_params(1, 2, 64, 300, 100)
    n = isa.rope_workspace_size(p)
    assert n == 300 * 32 * 8          # max(L_src, L_ctx) * D/2 (cos, sin) float pairs
    a = 1 << 20
    assert lib.isa_rope(ctypes.byref(p), 1.0, a, a, a, a, a, n, None) == 1
    assert b"base" in lib.isa_last_error()
    assert lib.isa_rope(ctypes.byref(p), float("inf"), a, a, a, a, a, n, None) == 1
    assert lib.isa_rope(ctypes.byref(p), 10000.0, a, a, a, None, a, n, None) == 1
    assert b"k_out is NULL" in lib.isa_last_error()
    assert lib.isa_rope(ctypes.byref(p), 10000.0, a, a + 8, a, a, a, n, None) == 1
    assert lib.isa_rope(ctypes.byref(p), 10000.0, a, a, a, a, a, n - 1, None) == 3


def test_debug_setters(isa):
    isa.set_wait_timeout_ns(1000)
    isa.set_wait_timeout_ns(0)
    isa.set_fault_injection(0)
    with pytest.raises(isa.IsaError):
        isa.set_fault_injection(7)


def test_backward_arguments_rejected_before_launch(isa):
    """isa_backward checks every pointer, the plan workspace and its own
    workspace on the host (fake device addresses: nothing may be launched)."""
    lib = isa.load_library()
    p = isa.make_params(1, 2, 64, 300, 100)
    n = isa.workspace_size(p)
    nb = isa.backward_workspace_size(p)
    BH, T, b, T_kv_pad = 2, 5 + 2, 64, 128
    # (lse*log2e, Delta) per padded block row, then dKc and dVc in fp32, each 256-byte aligned
    a256 = lambda x: (x + 255) // 256 * 256
    assert nb == a256(BH * T * b * 8) + 2 * a256(BH * T_kv_pad * 64 * 4)
    a = 1 << 20
    args = [ctypes.byref(p), a, a, a, a, n, a, a, a, a, a, a, a, nb, None]

    def call(**kw):
        x = list(args)
        for i, val in kw.items():
            x[int(i[1:])] = val
        return lib.isa_backward(*x)

    assert call(_8=None) == 1 and b"dout is NULL" in lib.isa_last_error()
    assert call(_10=a + 8) == 1 and b"dk" in lib.isa_last_error()
    assert call(_7=a + 2) == 1 and b"lse" in lib.isa_last_error()
    assert call(_12=a + 16) == 1 and b"backward workspace" in lib.isa_last_error()
    assert call(_13=nb - 1) == 3
    assert call(_5=n - 1) == 3


def test_coarse_residual_arguments_rejected_before_launch(isa):
    """isa_coarse_residual(_backward) check gamma, pointers and workspace
    sizes on the host (fake device addresses: nothing may be launched)."""
    lib = isa.load_library()
    p = isa.make_params(1, 2, 64, 300, 100)
    n = isa.workspace_size(p)
    nc = ctypes.c_size_t()
    assert lib.isa_coarse_residual_backward_workspace_size(ctypes.byref(p), ctypes.byref(nc)) == 0
    BH, T = 2, 5 + 2
    assert nc.value == (BH * T * 8 + 255) // 256 * 256 + BH * T * 64 * 4
    a = 1 << 20
    assert lib.isa_coarse_residual(ctypes.byref(p), float("nan"), a, n, a, None) == 1
    assert b"gamma" in lib.isa_last_error()
    assert lib.isa_coarse_residual(ctypes.byref(p), 1.0, a, n - 1, a, None) == 3
    assert lib.isa_coarse_residual(ctypes.byref(p), 1.0, a, n, a + 4, None) == 1
    args = [ctypes.byref(p), 1.0, a, n, a, a, a, a, None, a, nc.value, None]
    assert lib.isa_coarse_residual_backward(*(args[:4] + [None] + args[5:])) == 1
    assert b"dout is NULL" in lib.isa_last_error()
    assert lib.isa_coarse_residual_backward(*(args[:10] + [nc.value - 1] + args[11:])) == 3
    assert lib.isa_coarse_residual_backward(*(args[:8] + [a + 2] + args[9:])) == 1


def test_static_status_query_rejected_on_host(isa):
    """isa_forward_static_status refuses a NULL destination and a device on
    which isa_forward_static has not run, before any CUDA call."""
    lib = isa.load_library()
    assert lib.isa_forward_static_status(0, None, None) == isa.ISA_ERR_INVALID_ARG
    assert b"dst is NULL" in lib.isa_last_error()
    word = ctypes.c_int32(-1)
    assert lib.isa_forward_static_status(63, ctypes.addressof(word), None) == isa.ISA_ERR_INVALID_ARG
    assert b"has not run" in lib.isa_last_error()
    assert lib.isa_forward_static_status(-1, ctypes.addressof(word), None) == isa.ISA_ERR_INVALID_ARG
    assert word.value == -1
