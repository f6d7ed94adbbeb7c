"""The Python binding refuses host tensors and mismatched arguments before any
CUDA call (runs on a host without a GPU): every public forward/backward entry
raises FaError instead of falling back to another compute path.
"""

import pytest
import torch

from tiled_online_softmax_03_b200 import binding


def cpu(shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


QKV = [(1, 2, 64, 64), (1, 1, 64, 64), (1, 1, 64, 64)]


@pytest.mark.parametrize("call", [
    lambda q, k, v: binding.fa_fwd(q, k, v),
    lambda q, k, v: binding.fa_fwd_bias(q, k, v, cpu((1, 2, 64, 64))),
    lambda q, k, v: binding.fa_fwd_splitkv(q, k, v, 2),
    lambda q, k, v: binding.fa_fwd_splitkv_static(q, k, v, 2),
    lambda q, k, v: binding.fa_bwd(q, k, v, cpu((1, 2, 64, 64)), cpu((1, 2, 64), torch.float32),
                                   cpu((1, 2, 64, 64))),
    lambda q, k, v: binding.fa_fwd_fp8(q, k, v, 1.0, 1.0, 1.0),
])
def test_host_tensors_are_refused(call):
    q, k, v = (cpu(s) for s in QKV)
    with pytest.raises(binding.FaError):
        call(q, k, v)


def test_host_pipeline_refuses_mismatched_inputs():
    q = cpu((2, 2, 64, 64))
    with pytest.raises(binding.FaError, match="pinned"):
        binding.fa_fwd_from_host(q, cpu((2, 1, 64, 64)), cpu((2, 1, 64, 64)))
