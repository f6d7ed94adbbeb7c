"""fa_fwd_splitkv_static: split-KV on the library's static scratch, no allocation.

Collected last (file name) so it also runs after every other GPU test has used
the library; it passes alone too. Results are compared with fa_fwd_splitkv
(caller workspace) on the same inputs, on two calls in a row, within the
tolerances of the oracle comparisons.
"""

import pytest
import torch

from gpu_helpers import LSE_TOL, O_TOL
from tiled_online_softmax_03_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def inputs(B, Hq, Hk, N, d, dtype, causal, seed):
    w = Workload("t", B, Hq, Hk, N, d, dtype, causal, seed=seed)
    x = make_inputs(w)
    dev = torch.device("cuda:0")
    return w, tuple(x[n].to(dev) for n in ("q", "k", "v"))


def assert_close(a, b, dtype):
    (oa, la), (ob, lb) = a, b
    assert (oa.float() - ob.float()).abs().max().item() <= O_TOL[dtype]
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isfinite(la), fin)
    if fin.any():
        assert (la[fin] - lb[fin]).abs().max().item() <= LSE_TOL


@pytest.mark.parametrize("B,Hq,Hk,N,d,dtype,causal,splits", [
    (1, 4, 2, 1000, 128, "bf16", True, 3),
    (2, 2, 1, 777, 64, "fp16", False, 2),
    (1, 1, 1, 4096, 128, "bf16", False, 4),
])
def test_static_scratch_matches_caller_workspace_twice(B, Hq, Hk, N, d, dtype, causal, splits):
    from tiled_online_softmax_03_b200 import binding
    w, (q, k, v) = inputs(B, Hq, Hk, N, d, dtype, causal, seed=N + splits)
    assert binding.splitkv_workspace_bytes(B, Hq, N, d, splits) <= binding.STATIC_SCRATCH_BYTES
    ref = binding.fa_fwd_splitkv(q, k, v, splits, causal=causal)
    torch.cuda.synchronize()
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    for _ in range(2):  # two calls in a row on the same scratch
        o.fill_(7.0)
        lse.fill_(7.0)
        binding.fa_fwd_splitkv_static(q, k, v, splits, causal=causal, out=o, lse=lse)
        torch.cuda.synchronize()
        assert binding.device_status() == 0
        assert_close((o, lse), ref, w.torch_dtype)


def test_static_scratch_rejects_problems_beyond_its_size():
    from tiled_online_softmax_03_b200 import binding
    B, Hq, N, d, splits = 1, 8, 8192, 128, 4
    assert binding.splitkv_workspace_bytes(B, Hq, N, d, splits) > binding.STATIC_SCRATCH_BYTES
    _, (q, k, v) = inputs(B, Hq, Hq, N, d, "bf16", True, seed=5)
    with pytest.raises(binding.FaError, match="static scratch"):
        binding.fa_fwd_splitkv_static(q, k, v, splits, causal=True)
    # one split needs no scratch at all: the same problem runs
    o, lse = binding.fa_fwd_splitkv_static(q, k, v, 1, causal=True)
    torch.cuda.synchronize()
    ref = binding.fa_fwd(q, k, v, causal=True)
    assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1])
