"""fa_fwd_from_host: the forward on pinned host buffers, pipelined batch by
batch (copy in of b + 1, attention of b, copy out of b − 1 on three streams).
Each batch runs the same kernel on its slices, so the result must equal the
device-buffer fa_fwd bit for bit; the oracle comparison of fa_fwd itself is in
test_parity.py.
"""

import pytest
import torch

from tiled_online_softmax_03_b200.inputs import Workload, make_inputs


def _host_inputs(B, Hq, Hk, N, d, dtype, causal, lens=None, seed=0):
    w = Workload("h", B, Hq, Hk, N, d, dtype, causal, seed=seed)
    x = make_inputs(w)
    L = torch.tensor(lens, dtype=torch.int32) if lens is not None else None
    return w, x, L


def test_rejects_unpinned_or_device_inputs():
    from tiled_online_softmax_03_b200 import binding
    w, x, _ = _host_inputs(1, 2, 1, 64, 64, "fp16", False)
    with pytest.raises(binding.FaError, match="pinned"):
        binding.fa_fwd_from_host(x["q"], x["k"], x["v"])


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hq,Hk,N,d,dtype,causal,lens", [
    (3, 4, 2, 300, 128, "bf16", True, [300, 0, 170]),
    (2, 2, 2, 257, 64, "fp16", False, None),
    (1, 8, 1, 1000, 128, "bf16", True, [999]),
    (4, 4, 4, 129, 64, "bf16", True, None),
])
def test_equals_device_call_bitwise(B, Hq, Hk, N, d, dtype, causal, lens):
    from tiled_online_softmax_03_b200 import binding
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    w, x, L = _host_inputs(B, Hq, Hk, N, d, dtype, causal, lens, seed=N + B)
    dev = torch.device("cuda:0")
    o_ref, l_ref = binding.fa_fwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), causal=causal,
                                  key_pad_lens=L.to(dev) if L is not None else None)
    hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
    hL = L.pin_memory() if L is not None else None
    o, lse = binding.fa_fwd_from_host(hq, hk, hv, causal=causal, key_pad_lens=hL)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    assert torch.equal(o, o_ref.cpu()) and torch.equal(lse, l_ref.cpu())


@pytest.mark.gpu
def test_reused_buffers_across_calls():
    """Two calls in a row on one stream with the same device buffers and new
    inputs: the second result is that of the second inputs."""
    from tiled_online_softmax_03_b200 import binding
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dev = torch.device("cuda:0")
    B, Hq, Hk, N, d = 3, 4, 2, 384, 128
    bufs = {"q": torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=dev),
            "k": torch.empty((B, Hk, N, d), dtype=torch.bfloat16, device=dev),
            "v": torch.empty((B, Hk, N, d), dtype=torch.bfloat16, device=dev),
            "o": torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=dev),
            "lse": torch.empty((B, Hq, N), dtype=torch.float32, device=dev)}
    results = []
    for seed in (1, 2):
        w, x, _ = _host_inputs(B, Hq, Hk, N, d, "bf16", True, seed=seed)
        hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
        o, lse = binding.fa_fwd_from_host(hq, hk, hv, causal=True, device_buffers=bufs)
        results.append((x, o, lse))
    torch.cuda.synchronize()
    for x, o, lse in results:
        o_ref, l_ref = binding.fa_fwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), causal=True)
        assert torch.equal(o, o_ref.cpu()) and torch.equal(lse, l_ref.cpu())
