"""Backward (fa_bwd) against the float64 oracle's gradients.

The forward runs through fa_fwd (as a caller would), its O and LSE feed
fa_bwd, and dQ, dK, dV are compared with oracle.attention_backward evaluated
in float64 at the same 16-bit inputs (with the oracle's own exact O and LSE).

Tolerance, derived from the arithmetic rather than fixed: the kernel rounds P
and dS to the 16-bit type before its products (the tensor core takes no
other A operand) and its outputs once more. A plain 16-bit evaluation of the
same gradient — torch's math attention in that dtype, differentiated by
autograd on the CPU — makes the same kind of roundings, so the kernel's
largest error may be twice that evaluation's; or four half-ulps of the
dtype relative to the largest gradient entry (2^-7 bf16, 2^-10 fp16: one for
rounding the output, one for rounding dS, two for D = rowsum(dO ⊙ O) taken
from the 16-bit O and for the P rounding in dV), whichever is larger; with an
absolute floor of 2^-10 for gradients that vanish exactly (N = 1: P = 1 and
dS = 0 in exact arithmetic, so only rounding noise of D remains). A float32
emulation of these roundings on the CPU reproduces the kernel's dQ error on
the N = 300 case to the last bit (2.81e-3 of a largest entry of 0.52).
"""

import numpy as np
import pytest
import torch

from tiled_online_softmax_03_b200.inputs import WORKLOADS, Workload, make_inputs

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def problem(B, Hq, Hk, N, d, dtype, causal, lens=None, seed=0):
    w = Workload("t", B, Hq, Hk, N, d, dtype, causal, seed=seed)
    x = make_inputs(w)
    g = torch.Generator().manual_seed(seed + 99)
    x["dout"] = torch.randn((B, Hq, N, d), generator=g).to(w.torch_dtype)
    if lens is not None:
        x["key_pad_lens"] = torch.tensor(lens, dtype=torch.int32)
    return w, x


def run_gpu(w, x, scale=None):
    from tiled_online_softmax_03_b200 import binding
    scale = w.scale if scale is None else scale
    dev = torch.device("cuda:0")
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "dout"))
    lens = x["key_pad_lens"].to(dev) if x["key_pad_lens"] is not None else None
    o, lse = binding.fa_fwd(q, k, v, causal=w.causal, scale=scale, key_pad_lens=lens)
    dq, dk, dv = binding.fa_bwd(q, k, v, o, lse, do, causal=w.causal, scale=scale, key_pad_lens=lens)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    return dq, dk, dv


def reference(w, x, scale):
    lens = None if x["key_pad_lens"] is None else x["key_pad_lens"].tolist()
    q, k, v, do = (f64(x[n]) for n in ("q", "k", "v", "dout"))
    o, lse = oracle.attention(q, k, v, scale, w.causal, lens)
    return oracle.attention_backward(q, k, v, o, lse, do, scale, w.causal, lens)


def yardstick(w, x, scale):
    """Gradients of torch's math attention run in the 16-bit dtype on the CPU."""
    G = w.Hq // w.Hk
    q, k, v = (x[n].clone().requires_grad_() for n in ("q", "k", "v"))
    N = w.N
    L = [N] * w.B if x["key_pad_lens"] is None else [min(max(int(t), 0), N) for t in x["key_pad_lens"]]
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    mask = torch.stack([(j < l) & ((j <= i) if w.causal else (j >= 0)) for l in L])[:, None]
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        o = torch.nn.functional.scaled_dot_product_attention(
            q, k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1), attn_mask=mask,
            scale=scale)
    o = torch.nan_to_num(o)  # rows with no allowed key
    (o.float() * x["dout"].float()).sum().backward()
    return [torch.nan_to_num(t.grad).double().numpy() for t in (q, k, v)]


REL = {torch.bfloat16: 2.0 ** -7, torch.float16: 2.0 ** -10}


def bound_for(ref, yard, dtype):
    return max(2.0 * float(np.max(np.abs(yard - ref))), REL[dtype] * float(np.max(np.abs(ref))),
               2.0 ** -10)


def check(w, x, scale=None):
    scale = w.scale if scale is None else scale
    got = [f64(t) for t in run_gpu(w, x, scale)]
    ref = reference(w, x, scale)
    yard = yardstick(w, x, scale)
    for name, g, r, y in zip(("dq", "dk", "dv"), got, ref, yard):
        assert np.all(np.isfinite(g)), name
        err = float(np.max(np.abs(g - r))) if g.size else 0.0
        bound = bound_for(r, y, w.torch_dtype)
        assert err <= bound, f"{name}: max err {err:.3e} > bound {bound:.3e}"
    return got, ref


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp16", 64), ("bf16", 64), ("fp16", 128)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 300])
def test_backward_ragged_lengths(N, causal, dtype, d):
    w, x = problem(1, 2, 1, N, d, dtype, causal, seed=N)
    check(w, x)


@pytest.mark.parametrize("Hq,Hk", [(1, 1), (4, 4), (8, 2), (4, 1)])
def test_backward_head_groups(Hq, Hk):
    w, x = problem(2, Hq, Hk, 384, 128, "bf16", True, seed=Hq + Hk)
    check(w, x)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_key_padding(causal):
    w, x = problem(4, 2, 2, 400, 128, "bf16", causal, lens=[0, 1, 200, 400], seed=5)
    got, _ = check(w, x)
    assert not got[1][0].any() and not got[2][0].any() and not got[0][0].any()  # no key, no gradient


@pytest.mark.parametrize("scale", [0.0, -0.1, 0.3])
def test_backward_scale_values(scale):
    w, x = problem(1, 2, 1, 260, 64, "bf16", True, seed=7)
    got, _ = check(w, x, scale)
    if scale == 0.0:
        assert not got[0].any() and not got[1].any()  # dQ = dK = 0 exactly


def test_backward_several_tiles():
    w, x = problem(1, 4, 2, 1000, 128, "bf16", True, seed=8)
    check(w, x)


def test_backward_full_size_two_heads():
    """The 4K Llama shape: gradients of two heads against the oracle (the
    whole-problem gradient splits by head when Hq == Hk)."""
    w = WORKLOADS["llama7b_4k_causal"]
    x = make_inputs(w)
    g = torch.Generator().manual_seed(4242)
    x["dout"] = torch.randn(x["q"].shape, generator=g).to(w.torch_dtype)
    got = [f64(t) for t in run_gpu(w, x)]
    for h in (0, w.Hq - 1):
        sub = {n: x[n][:, h:h + 1] for n in ("q", "k", "v", "dout")}
        sub["key_pad_lens"] = None
        ws = w.with_(Hq=1, Hk=1)
        ref = reference(ws, sub, w.scale)
        yard = yardstick(ws, sub, w.scale)
        for gi, r, y in zip(got, ref, yard):
            gh = gi[:, h:h + 1]
            err = float(np.max(np.abs(gh - r)))
            bound = bound_for(r, y, w.torch_dtype)
            assert err <= bound, (h, err, bound)
