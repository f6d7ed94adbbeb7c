"""Additive bias (fa_fwd_bias) against the float64 oracle, element by element.

The oracle adds the same rounded 16-bit bias to its float64 scores
(S = scale·QKᵀ + bias, then the mask); tolerances are those of fa_fwd.
"""

import math

import numpy as np
import pytest
import torch

from gpu_helpers import O_TOL, compare, to64
from tiled_online_softmax_03_b200.inputs import WORKLOADS, Workload, make_bias, make_inputs

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def run(x, bias, causal, scale, lens=None):
    from tiled_online_softmax_03_b200 import binding
    dev = torch.device("cuda:0")
    o, lse = binding.fa_fwd_bias(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), bias.to(dev),
                                 causal=causal, scale=scale,
                                 key_pad_lens=None if lens is None else lens.to(dev))
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    return o, lse


def check(w, x, bias, lens=None):
    o, lse = run(x, bias, w.causal, w.scale, lens)
    o_ref, lse_ref = oracle.attention(to64(x["q"]), to64(x["k"]), to64(x["v"]), w.scale, w.causal,
                                      None if lens is None else lens.tolist(), bias=to64(bias))
    return compare(to64(o), to64(lse), o_ref, lse_ref, w.torch_dtype)


def small(B, Hq, Hk, N, d, dtype, causal, seed=0):
    w = Workload("t", B, Hq, Hk, N, d, dtype, causal, seed=seed)
    return w, make_inputs(w)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp16", 64), ("bf16", 64), ("fp16", 128)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [8, 136, 264, 520])
def test_bias_ragged_lengths(N, causal, dtype, d):
    w, x = small(2, 2, 1, N, d, dtype, causal, seed=N)
    check(w, x, make_bias(w, 2, 2))


@pytest.mark.parametrize("shape", [(1, 1), (1, 4), (2, 1), (2, 4)])
def test_bias_broadcast_shapes(shape):
    w, x = small(2, 4, 2, 384, 128, "bf16", True, seed=sum(shape))
    check(w, x, make_bias(w, *shape))


def test_bias_with_key_padding():
    w, x = small(4, 2, 2, 512, 128, "bf16", False, seed=5)
    lens = torch.tensor([0, 1, 200, 512], dtype=torch.int32)
    check(w, x, make_bias(w, 4, 1), lens)


def test_bias_large_values_force_rescales():
    """±30 offsets move the row max by far more than the rescale threshold."""
    w, x = small(1, 2, 2, 640, 128, "bf16", True, seed=6)
    check(w, x, make_bias(w, 1, 2, std=30.0))


def test_bias_minus_inf_masks_keys_and_empties_rows():
    """−inf entries remove keys; a row whose bias is −inf everywhere has no
    allowed key (O = 0, LSE = −inf, checked by compare)."""
    w, x = small(1, 2, 1, 256, 128, "fp16", False, seed=7)
    bias = make_bias(w, 1, 2)
    bias[0, 0, :, 100:] = -math.inf       # head 0: keys >= 100 removed
    bias[0, 1, 5, :] = -math.inf          # head 1, row 5: no allowed key at all
    check(w, x, bias)
    o, lse = run(x, bias, False, w.scale)
    assert torch.all(o[0, 1, 5] == 0) and lse[0, 1, 5].item() == -math.inf


def test_bias_zero_matches_fa_fwd():
    from tiled_online_softmax_03_b200 import binding
    w, x = small(2, 4, 2, 1000, 128, "bf16", True, seed=8)
    zero = torch.zeros(1, 1, 1000, 1000, dtype=torch.bfloat16)
    o1, l1 = run(x, zero, True, w.scale)
    o2, l2 = binding.fa_fwd(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), causal=True)
    assert (o1.float() - o2.float()).abs().max().item() <= O_TOL[torch.bfloat16]
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_bias_rejects_unsupported_n():
    from tiled_online_softmax_03_b200 import binding
    w, x = small(1, 1, 1, 100, 64, "bf16", False)
    with pytest.raises(binding.FaError, match="N % 8"):
        run(x, torch.zeros(1, 1, 100, 100, dtype=torch.bfloat16), False, w.scale)


def test_bias_full_size_sampled_rows():
    """4K Llama shape with a per-head bias [1, 32, 4096, 4096], sampled rows."""
    w = WORKLOADS["llama7b_4k_causal"]
    x = make_inputs(w)
    bias = make_bias(w, 1, w.Hq)
    o, lse = run(x, bias, True, w.scale)
    rng = np.random.default_rng(3)
    picks = sorted({(0, int(rng.integers(w.Hq)), int(i)) for i in
                    list(rng.integers(0, w.N, 60)) + [0, 127, 128, 4095]})
    o_ref = np.zeros((len(picks), w.d))
    l_ref = np.zeros(len(picks))
    for n, (b, h, i) in enumerate(picks):
        oo, ll = oracle.attention_rows(to64(x["q"][:, h:h + 1]), to64(x["k"][:, h:h + 1]),
                                       to64(x["v"][:, h:h + 1]), w.scale, True, None, [(0, 0, i)],
                                       bias=_row_bias(bias, h, i, w.N))
        o_ref[n], l_ref[n] = oo[0], ll[0]
    idx = tuple(np.array(picks).T)
    compare(to64(o)[idx], to64(lse)[idx], o_ref, l_ref, w.torch_dtype)


def _row_bias(bias, h, i, N):
    """A [1, 1, N, N] plane whose row i is the bias row (other rows unused)."""
    plane = np.zeros((1, 1, N, N))
    plane[0, 0, i] = to64(bias[0, h, i])
    return plane
