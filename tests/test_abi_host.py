"""Host-side checks of the C ABI (no GPU needed, no compute call made).

The library must load, export every function ``include/kda.h`` declares, and
reject bad arguments on the host before any CUDA call.
"""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# The argument-check tests pass made-up device addresses (0x1000 ...) and expect a refusal
# before any CUDA call.  Where a GPU is reachable, a regression in the check order could launch
# a kernel on such an address, so those tests run only where no device exists (the CPU suite).
host_only = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="made-up device addresses: run only where no GPU can be reached")


@pytest.fixture(scope="module")
def kda():
    from gated_delta_rule_73_b200 import build as B
    B.build()
    import gated_delta_rule_73_b200.kda as K
    return K


def _declared_functions():
    names = []
    for hdr in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not hdr.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", hdr)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\*?\s*(kda_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("kda_chunk_fwd", "kda_recurrent_step", "kda_chunk_fwd_prologue",
              "kda_recurrent_step_prologue", "kda_conv_state_from_prefill", "kda_chunk_fwd_gated",
              "kda_chunk_workspace_bytes", "kda_prologue_workspace_bytes", "kda_status_string",
              "kda_abi_version", "kda_chunk_bwd", "kda_chunk_bwd_workspace_bytes",
              "kda_segment_pair", "kda_segment_pair_workspace_bytes", "kda_affine_combine"):
        assert n in names


def test_library_exports_every_declared_symbol(kda):
    lib = ctypes.CDLL(kda.LIB_PATH)
    for n in _declared_functions():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_status_strings_and_version(kda):
    assert kda.kda_abi_version() == 110   # 1.10: the backward's workspace holds dS too
    for s in (0, -1, -2, -3, -4, -5, -6, -7):
        assert kda.status_string(s) and kda.status_string(s) != "unknown status"
    assert kda.status_string(-99) == "unknown status"


def _call_chunk(kda, ptr=0x1000, **kw):
    d = dict(B=1, T=64, H=2, dk=128, dv=128)
    d.update(kw.pop("dims", {}))
    opts = kw.pop("opts", kda.make_opts())
    p = [ctypes.c_void_p(ptr)] * 8
    for i, name in enumerate(("q", "k", "v", "g", "beta", "S0", "out", "S_T")):
        if name in kw:
            p[i] = ctypes.c_void_p(kw[name])
    return kda._lib.kda_chunk_fwd(*p, d["B"], d["T"], d["H"], d["dk"], d["dv"],
                                  ctypes.byref(opts), None)


@host_only
def test_chunk_fwd_rejects_bad_arguments_on_host(kda):
    # NULL required pointers
    assert _call_chunk(kda, q=0) == -1
    assert _call_chunk(kda, out=0) == -1
    # negative sizes
    assert _call_chunk(kda, dims=dict(T=-1)) == -1
    assert _call_chunk(kda, dims=dict(B=-2)) == -1
    # unsupported head dims
    assert _call_chunk(kda, dims=dict(dk=96)) == -4
    assert _call_chunk(kda, dims=dict(dv=256)) == -4
    # misaligned pointer (never dereferenced)
    assert _call_chunk(kda, k=0x1004) == -3
    # unknown flag bit / bad dtype / non-finite scale
    o = kda.make_opts(); o.flags = 64
    assert _call_chunk(kda, opts=o) == -1
    o = kda.make_opts(); o.flags = kda.KDA_QK_L2NORM | kda.KDA_FUSED | kda.KDA_SPLIT   # both paths forced
    assert _call_chunk(kda, opts=o) == -1
    o = kda.make_opts(); o.dtype = 7
    assert _call_chunk(kda, opts=o) == -1
    o = kda.make_opts(); o.scale = float("nan")
    assert _call_chunk(kda, opts=o) == -1
    # workspace missing for a shape that needs one
    assert _call_chunk(kda) == -7
    # overflowing sizes
    assert _call_chunk(kda, dims=dict(B=1, T=2**30, H=2**10)) == -2


@host_only
def test_empty_calls_are_noops(kda):
    # B == 0 or H == 0: nothing to do; T == 0 with S_T == NULL: nothing to write
    assert _call_chunk(kda, dims=dict(B=0)) == 0
    assert _call_chunk(kda, dims=dict(H=0)) == 0
    assert _call_chunk(kda, dims=dict(T=0), S_T=0) == 0


def test_workspace_sizes(kda):
    o = kda.make_opts()
    a = kda.kda_chunk_workspace_bytes(1, 64, 1, 128, 128, o)
    b = kda.kda_chunk_workspace_bytes(1, 128, 1, 128, 128, o)
    c = kda.kda_chunk_workspace_bytes(2, 65, 3, 128, 128, o)
    assert a >= 0 and b >= a and c >= b
    assert kda.kda_chunk_workspace_bytes(1, 0, 1, 128, 128, o) == 0
    assert kda.kda_chunk_workspace_bytes(1, 64, 1, 96, 128, o) == 0      # unsupported -> 0
    # FP32 path: the prologue's FP32 intermediates come first
    import torch
    f = kda.make_opts(torch.float32)
    p = kda.kda_prologue_workspace_bytes(1, 64, 2, 128, 128, f)
    assert p > 3 * 64 * 2 * 128 * 4
    # bf16 d=128, split form: the prologue runs inside the prep kernel, only records are needed
    split = kda.make_opts(torch.bfloat16, fused=False)
    assert (kda.kda_prologue_workspace_bytes(1, 64, 2, 128, 128, split)
            == kda.kda_chunk_workspace_bytes(1, 64, 2, 128, 128, split))
    # bf16 d=128, fused form: bf16 intermediates of the standalone prologue kernel
    fused = kda.make_opts(torch.bfloat16, fused=True)
    assert kda.kda_prologue_workspace_bytes(1, 64, 2, 128, 128, fused) >= 4 * 64 * 2 * 128 * 2


def test_workspace_follows_the_tensor_core_path(kda):
    """bf16 d=128: the split path needs one 74,240-byte record per chunk and head, the
    fused path none; without a flag the cost model picks the split form (with the two-group
    prep it is the faster one at every B*H; 148 SMs assumed without a GPU)."""
    import torch
    split = kda.make_opts(torch.bfloat16, fused=False)
    fused = kda.make_opts(torch.bfloat16, fused=True)
    auto = kda.make_opts(torch.bfloat16)
    nch = 3   # T = 130
    assert kda.kda_chunk_workspace_bytes(2, 130, 3, 128, 128, split) >= 2 * 3 * nch * 74240
    assert kda.kda_chunk_workspace_bytes(2, 130, 3, 128, 128, fused) == 0
    assert kda.kda_chunk_workspace_bytes(1, 4096, 16, 128, 128, auto) > 0
    if not torch.cuda.is_available():
        assert kda.kda_chunk_workspace_bytes(8, 8192, 32, 128, 128, auto) >= 8 * 32 * 128 * 74240


@host_only
def test_recurrent_step_rejects_bad_arguments_on_host(kda):
    vp = ctypes.c_void_p
    o = kda.make_opts()
    call = lambda ptrs, N=4, H=2, dk=128, dv=128: kda._lib.kda_recurrent_step(
        *[vp(p) for p in ptrs], N, H, dk, dv, ctypes.byref(o), None)
    good = [0x1000] * 7
    assert call([0] + good[1:]) == -1
    assert call(good[:5] + [0] + good[6:]) == -1          # S is required
    assert call(good[:2] + [0x1008] + good[3:]) == -3
    assert call(good, dk=32) == -4
    assert call(good, N=-1) == -1
    assert call(good, N=0) == 0


@host_only
def test_prologue_rejects_complex_and_unequal_dims(kda):
    vp = ctypes.c_void_p
    call = lambda opts, dk=128, dv=128: kda._lib.kda_chunk_fwd_prologue(
        *[vp(0x1000)] * 10, 1, 64, 2, dk, dv, ctypes.byref(opts), None)
    assert call(kda.make_opts(complex_gate=True)) == -4
    assert call(kda.make_opts(), dk=64, dv=128) == -4
    assert call(kda.make_opts()) == -7                     # needs a workspace


@host_only
def test_decode_prologue_rejects_bad_arguments_on_host(kda):
    """kda_recurrent_step_prologue / kda_conv_state_from_prefill argument checks (no GPU)."""
    P = 0x1000
    lib = kda._lib
    o = kda.make_opts()

    def step(N=2, H=3, dk=128, dv=128, opts=o, **kw):
        p = [ctypes.c_void_p(P)] * 10
        for i, name in enumerate(("q", "k", "v", "w", "cs", "z", "A", "b", "S", "out")):
            if name in kw:
                p[i] = ctypes.c_void_p(kw[name])
        return lib.kda_recurrent_step_prologue(*p, N, H, dk, dv, ctypes.byref(opts), None)

    assert step(dk=128, dv=64) == -4                 # needs dk == dv
    assert step(dk=96, dv=96) == -4
    c = kda.make_opts(complex_gate=True)
    assert step(opts=c) == -4                        # no signed-gate map for the prologue
    assert step(cs=0) == -1                          # conv state is required
    assert step(cs=0x1008) == -3                     # misaligned
    assert step(N=0) == 0 and step(H=0) == 0         # nothing to do

    def handoff(B=2, T=5, H=3, d=128, **kw):
        p = [ctypes.c_void_p(P)] * 4
        for i, name in enumerate(("q", "k", "v", "cs")):
            if name in kw:
                p[i] = ctypes.c_void_p(kw[name])
        return lib.kda_conv_state_from_prefill(*p, B, T, H, d, ctypes.byref(o), None)

    assert handoff(d=96) == -4
    assert handoff(T=-1) == -1
    assert handoff(cs=0) == -1
    assert handoff(B=0) == 0


@host_only
def test_unbounded_decay_flags_on_host(kda):
    """KDA_UNBOUNDED_DECAY / KDA_GATE_SOFTPLUS: only the split tensor-core form takes a gate
    without the -5 floor, so forcing a form is an argument error; the softplus map has no signed
    form.  bf16 d = 128 keeps the split form's workspace (its prep forms the diagonal blocks in
    FP32); with Complex-KDA, or fp32, the gate runs on the exact-FP32 path and its workspace."""
    import torch
    for fl in (kda.KDA_UNBOUNDED_DECAY, kda.KDA_GATE_SOFTPLUS):
        for forced in (kda.KDA_FUSED, kda.KDA_SPLIT):
            o = kda.make_opts(); o.flags = kda.KDA_QK_L2NORM | fl | forced
            assert _call_chunk(kda, opts=o) == -1
    o = kda.make_opts(complex_gate=True, gate_softplus=True)
    assert _call_chunk(kda, opts=o) == -1
    unb = kda.make_opts(torch.bfloat16, unbounded=True)
    sp = kda.make_opts(torch.bfloat16, gate_softplus=True)
    bounded = kda.make_opts(torch.bfloat16)
    unb_c = kda.make_opts(torch.bfloat16, unbounded=True, complex_gate=True)
    f32 = kda.make_opts(torch.float32)
    split = kda.kda_chunk_workspace_bytes(2, 130, 3, 128, 128, kda.make_opts(torch.bfloat16, fused=False))
    ref = kda.kda_chunk_workspace_bytes(2, 130, 3, 128, 128, f32)
    assert split > 0 and ref > 0 and split != ref
    assert kda.kda_chunk_workspace_bytes(2, 130, 3, 128, 128, unb) == split
    assert kda.kda_chunk_workspace_bytes(2, 130, 3, 128, 128, sp) == split
    assert kda.kda_chunk_workspace_bytes(2, 130, 3, 128, 128, bounded) == split
    assert kda.kda_chunk_workspace_bytes(2, 130, 3, 128, 128, unb_c) == ref
    # the prologue with the softplus gate is fused into the split form's prep: no intermediates
    assert kda.kda_prologue_workspace_bytes(2, 130, 3, 128, 128, sp) == split
    assert _call_chunk(kda, opts=unb) == -7                # still needs its workspace


@host_only
def test_chunk_bwd_host_checks(kda):
    """kda_chunk_bwd: argument checks before any CUDA call, and its workspace (FP32 states
    and state gradients every 8 tokens: 2*B*H*ceil(T/8)*dk*dv*4 bytes, 256-byte rounded)."""
    vp = ctypes.c_void_p
    o = kda.make_opts()

    def call(ptrs=None, B=1, T=64, H=2, dk=128, dv=128, opts=o):
        p = [vp(x) for x in (ptrs or [0x1000] * 14)]
        return kda._lib.kda_chunk_bwd(*p, B, T, H, dk, dv, ctypes.byref(opts), None)

    good = [0x1000] * 14
    assert call(good[:6] + [0] + good[7:]) == -1           # dout is required
    assert call(good[:8] + [0] + good[9:]) == -1           # grad_q is required
    assert call(good[:10] + [0x1004] + good[11:]) == -3    # misaligned grad_v
    assert call(dk=96) == -4
    assert call(T=-1) == -1
    assert call() == -7                                    # needs its workspace
    assert call(B=0) == 0
    assert call(good[:13] + [0], T=0) == 0                 # T = 0 without grad_S0: nothing to do
    bad = kda.make_opts(); bad.flags = 64
    assert call(opts=bad) == -1
    assert kda.kda_chunk_bwd_workspace_bytes(2, 33, 3, 128, 64, o) == 2 * 2 * 3 * 5 * 128 * 64 * 4
    assert kda.kda_chunk_bwd_workspace_bytes(1, 0, 3, 128, 128, o) == 0


@host_only
def test_segment_pair_and_combine_host_checks(kda):
    """kda_segment_pair / kda_affine_combine argument checks before any CUDA call, and the
    pair's workspace: zero v, identity start, scratch out, then the chunk workspace."""
    import torch
    vp = ctypes.c_void_p
    o = kda.make_opts(torch.float32)
    pair = lambda ptrs, T=64, dk=128, dv=128, opts=o: kda._lib.kda_segment_pair(
        *[vp(p) for p in ptrs], 1, T, 2, dk, dv, ctypes.byref(opts), None)
    good = [0x1000] * 7
    assert pair(good[:5] + [0] + good[6:]) == -1           # M_out required
    assert pair(good[:6] + [0x1008]) == -3                 # misaligned B_out
    assert pair(good, dk=96) == -4
    assert pair(good) == -7                                # needs a workspace
    ws = kda.kda_segment_pair_workspace_bytes(1, 64, 2, 128, 128, o)
    chunk = kda.kda_chunk_workspace_bytes(1, 64, 2, 128, 128, o)
    assert ws >= 64 * 2 * 128 * 4 + 2 * 128 * 128 * 4 + 64 * 2 * 128 * 4 + chunk
    comb = lambda M=0x1000, Bp=0x1000, n=2, S0=0x1000, out=0x1000, BH=3, dk=128, dv=128: \
        kda._lib.kda_affine_combine(vp(M), vp(Bp), n, vp(S0), vp(out), BH, dk, dv, None)
    assert comb(out=0) == -1
    assert comb(M=0) == -1
    assert comb(n=-1) == -1
    assert comb(dv=32) == -4
    assert comb(Bp=0x1004) == -3
    assert comb(BH=0) == 0


@host_only
def test_segment_forward_host_checks(kda):
    """kda_segment_forward: argument checks before any CUDA call.  On the split tensor-core
    form (bf16, d = 128) it needs the segment pair's workspace (the records and the identity
    start state) and out; the other configurations are kda_chunk_fwd and check as it does."""
    import torch
    vp = ctypes.c_void_p
    ob = kda.make_opts(torch.bfloat16)
    fwd = lambda ptrs, T=64, dk=128, dv=128, opts=ob: kda._lib.kda_segment_forward(
        *[vp(p) for p in ptrs], 1, T, 2, dk, dv, ctypes.byref(opts), None)
    good = [0x1000] * 8
    assert fwd(good[:6] + [0] + good[7:]) == -1            # out required
    assert fwd(good[:7] + [0x1008]) == -3                  # misaligned S_T
    assert fwd(good) == -7                                 # needs the pair's workspace
    pair_ws = kda.kda_segment_pair_workspace_bytes(1, 64, 2, 128, 128, ob)
    assert pair_ws > kda.kda_chunk_workspace_bytes(1, 64, 2, 128, 128, ob)   # records + identity
    small = kda.make_opts(torch.bfloat16)
    small.workspace, small.workspace_bytes = 0x10000, pair_ws - 16
    assert fwd(good, opts=small) == -7
    assert kda.kda_abi_version() >= 110
    # fp32: the whole chunk forward, with its own checks
    of = kda.make_opts(torch.float32)
    assert fwd(good, opts=of) == -7
    assert fwd(good, dk=96, opts=of) == -4


def test_binding_checks_shapes_before_any_call(kda):
    """The binding passes sizes read off q and v, so every other tensor must have the shape
    those sizes imply; a mismatch is refused (ValueError) before any pointer is taken."""
    import torch
    B, T, H, d = 1, 8, 2, 128
    q = torch.zeros(B, T, H, d, dtype=torch.bfloat16)
    good = dict(k=q, v=q, g=q, beta=torch.zeros(B, T, H, dtype=torch.bfloat16),
                S0=None, out=q, S_T=torch.zeros(B, H, d, d))
    o = kda.make_opts()
    for name, bad in (("k", torch.zeros(B, T, H, 64, dtype=torch.bfloat16)),
                      ("beta", torch.zeros(B, T, dtype=torch.bfloat16)),
                      ("S_T", torch.zeros(B, H, d, 64)),
                      ("out", torch.zeros(B, T + 1, H, d, dtype=torch.bfloat16))):
        args = dict(good, **{name: bad})
        with pytest.raises(ValueError, match=name):
            kda.kda_chunk_fwd(q, args["k"], args["v"], args["g"], args["beta"], args["S0"],
                              args["out"], args["S_T"], o)
    f = torch.float32
    grads = [torch.zeros(B, T, H, d), torch.zeros(B, T, H, d), torch.zeros(B, T, H, d),
             torch.zeros(B, T, H, d), torch.zeros(B, T, H), None]
    with pytest.raises(ValueError, match="grad_beta"):
        kda.kda_chunk_bwd(q, q, q, q, good["beta"], None, q, None, *grads[:4],
                          torch.zeros(B, T, H, 2), None, o)
    with pytest.raises(ValueError, match="M and Bp|M must"):
        kda.kda_affine_combine(torch.zeros(3, B * H, d, d), torch.zeros(2, B * H, d, d), 1, None,
                               torch.zeros(B * H, d, d))
