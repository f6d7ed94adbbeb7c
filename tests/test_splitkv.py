"""Split-KV forward (fa_fwd_splitkv) against the float64 oracle.

Cutting each Q tile pair's K/V range into chunks and merging the chunks by
log-sum-exp gives the full attention result (the oracle's merge_splits /
split_kv_attention are pinned to that on CPU), so the CUDA split path is
compared with the oracle's full attention under the same tolerances as fa_fwd.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import compare, oracle_full, oracle_rows, sample_picks, to64
from tiled_online_softmax_03_b200.inputs import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def run_split(x, causal, scale, splits, workspace=None):
    from tiled_online_softmax_03_b200 import binding
    dev = torch.device("cuda:0")
    lens = x["key_pad_lens"]
    o, lse = binding.fa_fwd_splitkv(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), splits,
                                    causal=causal, scale=scale,
                                    key_pad_lens=lens.to(dev) if lens is not None else None,
                                    workspace=workspace)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    return o, lse


def small(B, Hq, Hk, N, d, dtype, causal, lens=None, seed=0):
    w = Workload("t", B, Hq, Hk, N, d, dtype, causal, seed=seed)
    x = make_inputs(w)
    if lens is not None:
        x["key_pad_lens"] = torch.tensor(lens, dtype=torch.int32)
    return w, x


def check(w, x, splits):
    o, lse = run_split(x, w.causal, w.scale, splits)
    o_ref, lse_ref = oracle_full(x["q"], x["k"], x["v"], w.causal, w.scale, x["key_pad_lens"])
    return compare(to64(o), to64(lse), o_ref, lse_ref, w.torch_dtype)


@pytest.mark.parametrize("splits", [2, 3, 4, 7, 16])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "fp16")])
@pytest.mark.parametrize("N", [1, 129, 300, 1000])
def test_split_ragged_lengths(N, d, dtype, causal, splits):
    w, x = small(1, 4, 2, N, d, dtype, causal, seed=N + splits)
    check(w, x, splits)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("splits", [2, 5])
def test_split_key_padding_edges(causal, splits):
    lens = [0, 1, 127, 128, 129, 700, 1024, 2000]
    w, x = small(len(lens), 2, 1, 1024, 128, "bf16", causal, lens=lens, seed=3)
    check(w, x, splits)


@pytest.mark.parametrize("Hq,Hk", [(1, 1), (6, 2), (8, 1)])
def test_split_head_groups(Hq, Hk):
    w, x = small(2, Hq, Hk, 777, 128, "bf16", True, seed=Hq)
    check(w, x, 3)


def test_split_one_equals_fa_fwd_bitwise():
    from tiled_online_softmax_03_b200 import binding
    w, x = small(2, 4, 2, 600, 128, "bf16", True, seed=9)
    o1, l1 = run_split(x, True, w.scale, 1)
    dev = torch.device("cuda:0")
    o2, l2 = binding.fa_fwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_split_workspace_validation():
    from tiled_online_softmax_03_b200 import binding
    w, x = small(1, 2, 2, 256, 64, "bf16", False, seed=2)
    need = binding.splitkv_workspace_bytes(1, 2, 256, 64, 4)
    short = torch.empty(need - 1, dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.FaError, match="workspace"):
        run_split(x, False, w.scale, 4, workspace=short)
    big = torch.empty(need + 4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.FaError, match="aligned"):
        run_split(x, False, w.scale, 4, workspace=big[16:])
    # an exactly-sized workspace reused for two calls in a row
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    a = run_split(x, False, w.scale, 4, workspace=ws)
    b = run_split(x, False, w.scale, 4, workspace=ws)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("name,splits", [("llama7b_4k_causal", 2), ("long_32k_causal", 4)])
def test_split_full_size_sampled_rows(name, splits):
    w = WORKLOADS[name]
    x = make_inputs(w)
    o, lse = run_split(x, w.causal, w.scale, splits)
    picks = sample_picks(w.B, w.Hq, w.N, 120, seed=w.seed + splits)
    o_ref, lse_ref = oracle_rows(x["q"], x["k"], x["v"], w.causal, w.scale, x["key_pad_lens"],
                                 picks)
    idx = tuple(np.array(picks).T)
    compare(to64(o)[idx], to64(lse)[idx], o_ref, lse_ref, w.torch_dtype)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
