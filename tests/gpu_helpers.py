"""Helpers for the GPU parity tests: run the CUDA path, run the oracle, compare.

Tolerances are those the task states for this path: max |O − O_ref| <= 2e-2
for bf16 and 4e-3 for fp16, max |LSE − LSE_ref| <= 1e-3, with O_ref and
LSE_ref the float64 oracle on the same rounded inputs. Where LSE_ref is −inf
(a row with no allowed key) the kernel must give exactly −inf and O = 0.
"""

import numpy as np
import torch

import oracle

O_TOL = {torch.bfloat16: 2e-2, torch.float16: 4e-3}
LSE_TOL = 1e-3


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def run_cuda(q, k, v, causal, scale, lens, stream=None):
    from tiled_online_softmax_03_b200 import binding
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    ld = lens.to(dev) if lens is not None else None
    o, lse = binding.fa_fwd(qd, kd, vd, causal=causal, scale=scale, key_pad_lens=ld,
                            stream=stream)
    torch.cuda.synchronize()
    status = binding.device_status()
    assert status == 0, f"device status {status}"
    return o, lse


def oracle_full(q, k, v, causal, scale, lens):
    return oracle.attention(to64(q), to64(k), to64(v), scale, causal,
                            None if lens is None else lens.tolist())


def oracle_rows(q, k, v, causal, scale, lens, picks):
    """Oracle on selected rows; each (b, hq) slice is passed alone so only the
    needed heads are converted to float64."""
    G = q.shape[1] // k.shape[1]
    o = np.zeros((len(picks), v.shape[3]))
    lse = np.zeros(len(picks))
    groups = {}
    for n, (b, h, i) in enumerate(picks):
        groups.setdefault((b, h), []).append((n, i))
    for (b, h), items in groups.items():
        hk = h // G
        qs = to64(q[b:b + 1, h:h + 1])
        ks = to64(k[b:b + 1, hk:hk + 1])
        vs = to64(v[b:b + 1, hk:hk + 1])
        ls = None if lens is None else [int(lens[b])]
        oo, ll = oracle.attention_rows(qs, ks, vs, scale, causal, ls, [(0, 0, i) for _, i in items])
        for (n, _), orow, lrow in zip(items, oo, ll):
            o[n], lse[n] = orow, lrow
    return o, lse


def compare(o_gpu, lse_gpu, o_ref, lse_ref, dtype):
    """Assert the tolerances; return (max O error, max LSE error)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), empty), "rows with no allowed key differ"
    assert np.all(np.isfinite(o_gpu)), "non-finite output"
    if empty.any():
        assert np.all(o_gpu[empty] == 0.0), "O of an empty row is not 0"
    o_err = float(np.max(np.abs(o_gpu - o_ref))) if o_gpu.size else 0.0
    fin = ~empty
    lse_err = float(np.max(np.abs(lse_gpu[fin] - lse_ref[fin]))) if fin.any() else 0.0
    assert o_err <= O_TOL[dtype], f"max |dO| = {o_err:.3e} > {O_TOL[dtype]:.0e}"
    assert lse_err <= LSE_TOL, f"max |dLSE| = {lse_err:.3e} > {LSE_TOL:.0e}"
    return o_err, lse_err


def sample_picks(B, Hq, N, n_rows, seed, extra_rows=()):
    """Rows spread over batch, heads and positions, plus the first/last rows and
    rows around tile boundaries."""
    rng = np.random.default_rng(seed)
    picks = set()
    for _ in range(n_rows):
        picks.add((int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(N))))
    for i in (0, 1, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1) + tuple(extra_rows):
        if 0 <= i < N:
            picks.add((int(rng.integers(B)), int(rng.integers(Hq)), i))
    picks.add((0, 0, 0))
    picks.add((B - 1, Hq - 1, N - 1))
    return sorted(picks)
