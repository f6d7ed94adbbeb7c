"""CUDA path (through the C ABI) against the float64 oracle, element by element.

Small problems are compared on every output; the full-size workloads are
compared on sampled rows that the oracle computes one by one, in the same
launch configuration the benchmark times.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import (LSE_TOL, O_TOL, compare, oracle_full, oracle_rows, run_cuda,
                         sample_picks, to64)
from tiled_online_softmax_03_b200.inputs import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def small(B, Hq, Hk, N, d, dtype, causal, lens=None, seed=0, qk_mult=1.0):
    w = Workload("t", B, Hq, Hk, N, d, dtype, causal, qk_mult=qk_mult, seed=seed)
    x = make_inputs(w)
    if lens is not None:
        x["key_pad_lens"] = torch.tensor(lens, dtype=torch.int32)
    return w, x


def check_full(w, x, scale=None):
    scale = w.scale if scale is None else scale
    o, lse = run_cuda(x["q"], x["k"], x["v"], w.causal, scale, x["key_pad_lens"])
    o_ref, lse_ref = oracle_full(x["q"], x["k"], x["v"], w.causal, scale, x["key_pad_lens"])
    return compare(to64(o), to64(lse), o_ref, lse_ref, w.torch_dtype)


# ------------------------------------------------------------- small shapes

@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 127, 128, 129, 300, 513])
def test_ragged_lengths(N, causal, d, dtype):
    w, x = small(1, 2, 1, N, d, dtype, causal, seed=N + 7 * d)
    check_full(w, x)


@pytest.mark.parametrize("Hq,Hk", [(1, 1), (2, 2), (4, 2), (8, 2), (6, 2), (3, 1), (32, 1), (8, 8)])
@pytest.mark.parametrize("causal", [False, True])
def test_head_groups(Hq, Hk, causal):
    w, x = small(2, Hq, Hk, 384, 128, "bf16", causal, seed=Hq * 10 + Hk)
    check_full(w, x)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("N", [1000, 1024])
def test_one_query_head_per_kv_head_several_units_per_cta(N, dtype):
    # 40 heads × 4 tile pairs = 480 units on at most 148 CTAs: each CTA walks
    # several units whose tile 0 ends one K/V tile before tile 1 (the next
    # unit's first S is issued during that last tile)
    w, x = small(3, 40, 40, N, 128, dtype, True, seed=N)
    check_full(w, x)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_key_padding_edges(causal, d):
    # lengths 0 (every row empty), 1, a tile edge, ragged, and N itself
    lens = [0, 1, 128, 200, 384, 383]
    w, x = small(len(lens), 4, 2, 384, d, "bf16", causal, lens=lens, seed=3 + d)
    check_full(w, x)


@pytest.mark.parametrize("scale", [0.0, -0.2, 0.5])
def test_scale_values(scale):
    w, x = small(1, 2, 2, 300, 64, "fp16", True, seed=11)
    check_full(w, x, scale=scale)


def test_peaked_rows_stress_rescale():
    # Q, K scaled by 3 (the long-context recipe) at a size the oracle finishes quickly
    w, x = small(1, 4, 2, 1024, 128, "bf16", True, seed=5, qk_mult=3.0)
    check_full(w, x)


def test_increasing_scores_force_every_rescale():
    # scores grow along the key axis, so the running max moves on every K/V tile
    w, x = small(1, 1, 1, 1024, 64, "bf16", False, seed=9)
    ramp = torch.linspace(-30, 30, 1024).reshape(1, 1, 1024, 1)
    x["k"] = (torch.zeros(1, 1, 1024, 64) + ramp / 8).to(torch.bfloat16)
    x["q"] = torch.ones(1, 1, 1024, 64, dtype=torch.bfloat16)
    check_full(w, x)


# ------------------------------------------------------- the five workloads

def test_single_head_128_full():
    w = WORKLOADS["single_head_128"]
    _report(w.name, "every element", check_full(w, make_inputs(w)), w.torch_dtype)


def test_bert_large_512_keypad_full():
    w = WORKLOADS["bert_large_512_keypad"]
    _report(w.name, "every element", check_full(w, make_inputs(w)), w.torch_dtype)


def _full_size_run(name):
    w = WORKLOADS[name]
    x = make_inputs(w)
    o, lse = run_cuda(x["q"], x["k"], x["v"], w.causal, w.scale, x["key_pad_lens"])
    # properties that hold at any size: finite everywhere, causal row 0 is V row 0
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    G = w.Hq // w.Hk
    v0 = x["v"][:, torch.arange(w.Hq) // G, 0].to(o.device)
    assert torch.equal(o[:, :, 0], v0)
    return w, x, o, lse


def _report(name, part, errs, dtype):
    o_err, lse_err = errs
    tol = O_TOL[dtype]
    print(f"PARITY {name} {part}: max|dO| {o_err:.4e} (bound {tol:.0e}, margin {tol - o_err:.4e}) "
          f"max|dLSE| {lse_err:.4e} (bound {LSE_TOL:.0e})")


@pytest.mark.parametrize("name", ["llama7b_4k_causal", "gqa_8k_causal", "mqa_8k_causal",
                                  "long_32k_causal"])
def test_full_size_sampled_rows(name):
    """The full workload in the launch configuration the benchmark times;
    compared on rows spread over the whole output, and on the 256 rows with
    the largest max |O| (the rows closest to the bf16 bound: peaked rows
    whose O is nearly one V row). The rows are chosen from the kernel's
    output; their expected values come from the oracle alone."""
    w, x, o, lse = _full_size_run(name)
    picks = set(sample_picks(w.B, w.Hq, w.N, 160, seed=w.seed))
    amax = o.abs().amax(-1).flatten()
    top = torch.topk(amax.float(), 256).indices.cpu().numpy()
    for f in top:
        b, rem = divmod(int(f), w.Hq * w.N)
        h, i = divmod(rem, w.N)
        picks.add((b, h, i))
    picks = sorted(picks)
    o_ref, lse_ref = oracle_rows(x["q"], x["k"], x["v"], w.causal, w.scale, x["key_pad_lens"],
                                 picks)
    idx = tuple(np.array(picks).T)
    errs = compare(to64(o)[idx], to64(lse)[idx], o_ref, lse_ref, w.torch_dtype)
    _report(name, f"{len(picks)} sampled + largest-|O| rows", errs, w.torch_dtype)


@pytest.mark.parametrize("name", ["gqa_8k_causal", "mqa_8k_causal", "long_32k_causal"])
def test_full_size_whole_head(name):
    """One whole (b, hq) head of the full workload, every element, against the
    oracle on that head; and every tile-edge row (the last and first row of
    each 128-row Q tile) of a second head from another batch."""
    w, x, o, lse = _full_size_run(name)
    G = w.Hq // w.Hk
    b, h = w.B - 1, w.Hq // 2 + 1
    hk = h // G
    o_ref, lse_ref = oracle_full(x["q"][b:b + 1, h:h + 1], x["k"][b:b + 1, hk:hk + 1],
                                 x["v"][b:b + 1, hk:hk + 1], w.causal, w.scale, None)
    errs = compare(to64(o[b:b + 1, h:h + 1]), to64(lse[b:b + 1, h:h + 1]), o_ref, lse_ref,
                   w.torch_dtype)
    _report(name, f"whole head (b={b}, hq={h})", errs, w.torch_dtype)
    b2, h2 = 0, w.Hq - 1
    edges = sorted({r for t in range(0, w.N, 128) for r in (t - 1, t) if 0 <= r < w.N} | {w.N - 1})
    picks = [(b2, h2, i) for i in edges]
    o_ref, lse_ref = oracle_rows(x["q"], x["k"], x["v"], w.causal, w.scale, x["key_pad_lens"],
                                 picks)
    idx = tuple(np.array(picks).T)
    errs = compare(to64(o)[idx], to64(lse)[idx], o_ref, lse_ref, w.torch_dtype)
    _report(name, f"{len(picks)} tile-edge rows of (b={b2}, hq={h2})", errs, w.torch_dtype)


@pytest.mark.parametrize("splits", [1, 2])
def test_head_grouped_order_with_key_padding(splits):
    """The 8K GQA shape runs the head-grouped unit order on a B200 (three
    groups); here with per-sequence key lengths (full, ragged, one key, none)
    and, with splits = 2, through split-KV, whose grouped order deals out
    chunk pairs. Sampled rows and every row around the ragged length."""
    from tiled_online_softmax_03_b200 import binding
    w = WORKLOADS["gqa_8k_causal"]
    props = torch.cuda.get_device_properties(0)
    grid = min(binding.num_units(w.B, w.Hq, w.Hk, w.N, 1), props.multi_processor_count)
    assert binding.unit_groups(w.B, w.Hq, w.Hk, w.N, w.d, 1, grid, props.L2_cache_size) > 1
    x = make_inputs(w)
    lens = torch.tensor([w.N, 5000, 1, 0], dtype=torch.int32)
    dev = torch.device("cuda:0")
    q, k, v, ld = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), lens.to(dev)
    if splits == 1:
        o, lse = binding.fa_fwd(q, k, v, causal=True, scale=w.scale, key_pad_lens=ld)
    else:
        o, lse = binding.fa_fwd_splitkv(q, k, v, splits, causal=True, scale=w.scale, key_pad_lens=ld)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    picks = set(sample_picks(w.B, w.Hq, w.N, 120, seed=w.seed + splits))
    for i in (4990, 4999, 5000, 5001, 5119, 5120, w.N - 1):
        picks.add((1, 3, i))
    for i in (0, 1, 200, w.N - 1):
        picks.update({(2, 7, i), (3, 30, i)})
    picks = sorted(picks)
    o_ref, lse_ref = oracle_rows(x["q"], x["k"], x["v"], True, w.scale, lens, picks)
    idx = tuple(np.array(picks).T)
    errs = compare(to64(o)[idx], to64(lse)[idx], o_ref, lse_ref, w.torch_dtype)
    _report(w.name, f"key lengths {lens.tolist()}, splits {splits}: {len(picks)} rows", errs,
            w.torch_dtype)


def test_llama7b_4k_full():
    """The Llama-7B-shaped workload (B=1, 32 heads, N=4096, fp16, causal) in
    the launch configuration the benchmark times, every element of O and LSE
    against the float64 oracle, one head at a time (~0.5 s of oracle per head)."""
    w = WORKLOADS["llama7b_4k_causal"]
    x = make_inputs(w)
    o, lse = run_cuda(x["q"], x["k"], x["v"], w.causal, w.scale, None)
    o64, lse64 = to64(o), to64(lse)
    worst_o, worst_lse = 0.0, 0.0
    for h in range(w.Hq):
        o_ref, lse_ref = oracle_full(x["q"][:, h:h + 1], x["k"][:, h:h + 1], x["v"][:, h:h + 1],
                                     True, w.scale, None)
        eo, el = compare(o64[:, h:h + 1], lse64[:, h:h + 1], o_ref, lse_ref, w.torch_dtype)
        worst_o, worst_lse = max(worst_o, eo), max(worst_lse, el)
    _report(w.name, f"all {w.Hq} heads, every element", (worst_o, worst_lse), w.torch_dtype)


# -------------------------------------------------------------- exact cases

@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_causal_row0_is_exact(dtype):
    w, x = small(2, 4, 2, 777, 128, dtype, True, seed=21)
    o, lse = run_cuda(x["q"], x["k"], x["v"], True, w.scale, None)
    G = 2
    v0 = x["v"][:, torch.arange(4) // G, 0].to(o.device)
    assert torch.equal(o[:, :, 0], v0)
    s00 = w.scale * (to64(x["q"][:, :, 0]) * to64(x["k"][:, torch.arange(4) // G, 0])).sum(-1)
    assert np.max(np.abs(to64(lse[:, :, 0]) - s00)) < 1e-4


def test_single_key_rows_are_exact():
    lens = [1, 1]
    w, x = small(2, 2, 1, 256, 64, "bf16", False, lens=lens, seed=4)
    o, _ = run_cuda(x["q"], x["k"], x["v"], False, w.scale, x["key_pad_lens"])
    want = x["v"][:, [0, 0], 0:1].expand(2, 2, 256, 64).to(o.device)
    assert torch.equal(o, want)


def test_uniform_v_is_reproduced():
    w, x = small(1, 2, 2, 640, 128, "bf16", True, seed=8)
    row = torch.randn(128).to(torch.bfloat16)
    x["v"] = row.expand(1, 2, 640, 128).contiguous()
    o, _ = run_cuda(x["q"], x["k"], x["v"], True, w.scale, None)
    err = (o.float().cpu() - row.float()).abs().max().item()
    ulp = row.float().abs().max().item() * 2 ** -7
    assert err <= ulp


def test_deterministic_and_stream():
    w, x = small(2, 8, 2, 1000, 128, "bf16", True, seed=1)
    o1, l1 = run_cuda(x["q"], x["k"], x["v"], True, w.scale, None)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o2, l2 = run_cuda(x["q"], x["k"], x["v"], True, w.scale, None,
                          stream=s.cuda_stream)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_same_addresses_new_shapes():
    """Calls that pass the same buffer addresses with other extents (the
    library keeps recently encoded tensor maps per address, type and extents)
    give each shape's own result."""
    dev = torch.device("cuda:0")
    big = torch.empty(4 * 8 * 1024 * 128, dtype=torch.bfloat16, device=dev)
    kbig, vbig, obig = (torch.empty_like(big) for _ in range(3))
    results = []
    for (B, Hq, Hk, N) in [(2, 4, 2, 1024), (4, 8, 2, 512), (1, 2, 1, 2048), (2, 4, 2, 1024)]:
        w, x = small(B, Hq, Hk, N, 128, "bf16", True, seed=B * 100 + N)
        q = big[:B * Hq * N * 128].view(B, Hq, N, 128)
        k = kbig[:B * Hk * N * 128].view(B, Hk, N, 128)
        v = vbig[:B * Hk * N * 128].view(B, Hk, N, 128)
        q.copy_(x["q"]); k.copy_(x["k"]); v.copy_(x["v"])
        o = obig[:B * Hq * N * 128].view(B, Hq, N, 128)
        from tiled_online_softmax_03_b200 import binding
        _, lse = binding.fa_fwd(q, k, v, causal=True, out=o)
        torch.cuda.synchronize()
        o_ref, lse_ref = run_cuda(x["q"], x["k"], x["v"], True, w.scale, None)  # fresh buffers
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        results.append(o.clone())
    assert torch.equal(results[0], results[3])
