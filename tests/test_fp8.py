"""FP8 (E4M3) forward (fa_fwd_fp8) against the float64 oracle.

Inputs are N(0,1) samples quantised per tensor to E4M3 (descale = amax/448);
the oracle runs on the decoded values (every E4M3 value times its descale is
exact in float64), so it is the exact attention of the kernel's inputs.

Tolerance, derived from the arithmetic: the kernel rounds P to E4M3 for the
P·V product (3 mantissa bits; values below 2^-9 flush to zero) and divides by
the sum of the rounded P. A float64 evaluation that makes only that rounding —
P = exp(S − rowmax) rounded to E4M3 to nearest even, O = Σ P̃ V / Σ P̃ — is the
yardstick: the kernel's largest O error may be at most twice the yardstick's
plus the bfloat16 rounding of O (2^-8 of its largest entry). The kernel's P is
taken against a running reference max that lags the row max by up to 2^8, so
its values are larger and flush less than the yardstick's. LSE does not pass
through the 8-bit rounding: it keeps the fa_fwd bound of 1e-3.
"""


import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

FP8 = getattr(torch, "float8_e4m3fn", None)
LSE_TOL = 1e-3


@pytest.fixture(autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def quantise(x):
    """Per-tensor E4M3: returns (fp8 tensor, descale)."""
    amax = float(x.abs().max())
    descale = amax / 448.0 if amax > 0 else 1.0
    return (x / descale).to(FP8), descale


def make(B, Hq, Hk, N, d, causal, lens=None, seed=0, qk_mult=1.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, N, d), generator=g) * qk_mult
    k = torch.randn((B, Hk, N, d), generator=g) * qk_mult
    v = torch.randn((B, Hk, N, d), generator=g)
    (q8, qs), (k8, ks), (v8, vs) = quantise(q), quantise(k), quantise(v)
    L = None if lens is None else torch.tensor(lens, dtype=torch.int32)
    return dict(q8=q8, k8=k8, v8=v8, qs=qs, ks=ks, vs=vs, lens=L, causal=causal, d=d)


def decoded(x):
    return [x["q8"].double().numpy() * x["qs"], x["k8"].double().numpy() * x["ks"],
            x["v8"].double().numpy() * x["vs"]]


def run(x, scale):
    from tiled_online_softmax_03_b200 import binding
    dev = torch.device("cuda:0")
    lens = x["lens"].to(dev) if x["lens"] is not None else None
    o, lse = binding.fa_fwd_fp8(x["q8"].to(dev), x["k8"].to(dev), x["v8"].to(dev), x["qs"], x["ks"],
                                x["vs"], causal=x["causal"], scale=scale, key_pad_lens=lens)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


def e4m3_round(p):
    return torch.from_numpy(np.asarray(p, dtype=np.float32)).to(FP8).double().numpy()


def yardstick(q, k, v, scale, causal, lens, rows=None):
    """O with only the E4M3 rounding of P (against the exact row max), for all
    rows or the given row indices (then [B, Hq, len(rows), d])."""
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    o = np.zeros((B, Hq, len(rows), d))
    for b in range(B):
        L = N if lens is None else min(max(int(lens[b]), 0), N)
        ok = oracle.allowed_keys(rows, N, causal, L)
        for h in range(Hq):
            s = oracle.scores(q[b, h, rows], k[b, h // G], scale, ok)
            m = s.max(axis=1)
            has = np.isfinite(m)
            p = np.zeros_like(s)
            p[has] = np.exp(s[has] - m[has][:, None])
            pq = e4m3_round(p)
            den = pq.sum(axis=1)
            good = den > 0
            o[b, h][good] = (pq[good] @ v[b, h // G]) / den[good][:, None]
    return o


def check(x, scale=None):
    d = x["d"]
    scale = d ** -0.5 if scale is None else scale
    o, lse = run(x, scale)
    q, k, v = decoded(x)
    lens = None if x["lens"] is None else x["lens"].tolist()
    o_ref, lse_ref = oracle.attention(q, k, v, scale, x["causal"], lens)
    o_y = yardstick(q, k, v, scale, x["causal"], lens)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty)
    assert np.all(np.isfinite(o)) and np.all(o[empty] == 0)
    err = float(np.max(np.abs(o - o_ref)))
    bound = 2.0 * float(np.max(np.abs(o_y - o_ref))) + 2.0 ** -8 * float(np.max(np.abs(o_ref)))
    assert err <= bound, f"max |dO| {err:.3e} > {bound:.3e}"
    fin = ~empty
    if fin.any():
        lerr = float(np.max(np.abs(lse[fin] - lse_ref[fin])))
        assert lerr <= LSE_TOL, f"max |dLSE| {lerr:.3e}"
    return err, bound


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [16, 144, 256, 1008])
def test_fp8_lengths(N, causal):
    check(make(1, 2, 1, N, 128, causal, seed=N))


@pytest.mark.parametrize("Hq,Hk", [(4, 4), (8, 2), (4, 1)])
def test_fp8_head_groups(Hq, Hk):
    check(make(2, Hq, Hk, 384, 128, True, seed=Hq * 10 + Hk))


def test_fp8_key_padding():
    check(make(4, 2, 2, 512, 128, False, lens=[0, 1, 200, 512], seed=5))


def test_fp8_peaked_scores():
    """Q, K ×3: row maxima move often (rescales) and P spans the E4M3 range."""
    check(make(1, 2, 2, 640, 128, True, seed=6, qk_mult=3.0))


def test_fp8_unsupported_shapes():
    from tiled_online_softmax_03_b200 import binding
    x = make(1, 1, 1, 100, 128, False)
    with pytest.raises(binding.FaError, match="N % 16"):
        run(x, 0.1)
    x = make(1, 1, 1, 128, 64, False)
    with pytest.raises(binding.FaError, match="head dim"):
        run(x, 0.1)


def test_fp8_full_size_sampled_rows():
    """The 8K GQA shape in FP8, sampled rows of two heads against the oracle."""
    B, Hq, Hk, N, d = 4, 32, 8, 8192, 128
    x = make(B, Hq, Hk, N, d, True, seed=1003)
    o, lse = run(x, d ** -0.5)
    q, k, v = decoded(x)
    rng = np.random.default_rng(9)
    for (b, h) in [(0, 0), (B - 1, Hq - 1)]:
        rows = sorted({int(i) for i in rng.integers(0, N, 24)} | {0, 127, 128, N - 1})
        picks = [(0, 0, i) for i in rows]
        hk = h // (Hq // Hk)
        qs, ks, vs = q[b:b + 1, h:h + 1], k[b:b + 1, hk:hk + 1], v[b:b + 1, hk:hk + 1]
        o_ref, l_ref = oracle.attention_rows(qs, ks, vs, d ** -0.5, True, None, picks)
        o_y = yardstick(qs, ks, vs, d ** -0.5, True, None, rows)[0, 0]
        err = float(np.max(np.abs(o[b, h][rows] - o_ref)))
        bound = 2.0 * float(np.max(np.abs(o_y - o_ref))) + 2.0 ** -8 * float(np.max(np.abs(o_ref)))
        assert err <= bound, (b, h, err, bound)
        assert float(np.max(np.abs(lse[b, h][rows] - l_ref))) <= LSE_TOL
