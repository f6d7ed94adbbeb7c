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


@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 6, 31, 32, 33])
@pytest.mark.parametrize("chunks", [None, 1, 2, 3, 100])
def test_chunk_ranges_partition_the_batch(B, chunks):
    from tiled_online_softmax_03_b200.binding import chunk_ranges
    r = chunk_ranges(B, chunks)
    assert r[0][0] == 0 and r[-1][1] == B
    assert all(a1 == b0 for (_, a1), (b0, _) in zip(r, r[1:]))
    sizes = [b1 - b0 for b0, b1 in r]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    assert len(r) == (min(B, 4) if chunks is None else min(chunks, B))


@pytest.mark.gpu
@pytest.mark.parametrize("chunks", [None, 1, 3, 6])
def test_multi_batch_chunks_equal_device_call(chunks):
    from tiled_online_softmax_03_b200 import binding
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B, Hq, Hk, N, d = 6, 4, 2, 200, 64
    w, x, L = _host_inputs(B, Hq, Hk, N, d, "bf16", False, [200, 0, 7, 128, 129, 55], seed=11)
    dev = torch.device("cuda:0")
    o_ref, l_ref = binding.fa_fwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), key_pad_lens=L.to(dev))
    hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
    o, lse = binding.fa_fwd_from_host(hq, hk, hv, key_pad_lens=L.pin_memory(), chunks=chunks)
    torch.cuda.synchronize()
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


class _FakeDev:
    """Stands in for a CUDA tensor in the host-side argument checks."""

    def __init__(self, shape, dtype, device="cuda:0", contiguous=True):
        self.shape = tuple(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self.is_cuda = self.device.type == "cuda"
        self._c = contiguous

    def is_contiguous(self):
        return self._c


class _Pinned:
    """A CPU tensor that reports itself page-locked (no CUDA on this host)."""

    def __init__(self, t):
        self.t = t
        self.shape, self.dtype, self.is_cuda = t.shape, t.dtype, False

    def __getattr__(self, name):
        return getattr(self.t, name)

    def is_pinned(self):
        return True

    def dim(self):
        return self.t.dim()

    def numel(self):
        return self.t.numel()

    def is_contiguous(self):
        return True


def _buffers(B, Hq, Hk, N, d, dt, lens=True, **override):
    bufs = {"q": _FakeDev((B, Hq, N, d), dt), "k": _FakeDev((B, Hk, N, d), dt),
            "v": _FakeDev((B, Hk, N, d), dt), "o": _FakeDev((B, Hq, N, d), dt),
            "lse": _FakeDev((B, Hq, N), torch.float32),
            "lens": _FakeDev((B,), torch.int32) if lens else None}
    bufs.update(override)
    return bufs


@pytest.mark.parametrize("bad", [
    {"o": _FakeDev((2, 4, 100, 64), torch.float16)},              # wrong head count
    {"lse": _FakeDev((2, 2, 100), torch.float16)},                # wrong dtype
    {"k": _FakeDev((2, 1, 100, 64), torch.bfloat16, "cuda:1")},   # other device
    {"v": _FakeDev((2, 1, 100, 64), torch.bfloat16, contiguous=False)},
    {"lens": None},                                              # padding without a buffer
])
def test_device_buffer_checks(bad):
    from tiled_online_softmax_03_b200 import binding
    B, Hq, Hk, N, d = 2, 2, 1, 100, 64
    dt = torch.bfloat16
    q, k, v = (_Pinned(torch.zeros(s, dtype=dt)) for s in [(B, Hq, N, d), (B, Hk, N, d), (B, Hk, N, d)])
    out, lse = _Pinned(torch.zeros((B, Hq, N, d), dtype=dt)), _Pinned(torch.zeros((B, Hq, N)))
    lens = _Pinned(torch.zeros(B, dtype=torch.int32))
    with pytest.raises(binding.FaError, match="device_buffers"):
        binding.fa_fwd_from_host(q, k, v, key_pad_lens=lens, out=out, lse=lse,
                                 device_buffers=_buffers(B, Hq, Hk, N, d, dt, **bad),
                                 device=torch.device("cuda", 0))
    # the buffers the benchmark passes get past every check (up to the first
    # CUDA call, which this host cannot make)
    with pytest.raises(Exception) as e:
        binding.fa_fwd_from_host(q, k, v, key_pad_lens=lens, out=out, lse=lse,
                                 device_buffers=_buffers(B, Hq, Hk, N, d, dt),
                                 device=torch.device("cuda", 0))
    assert not isinstance(e.value, binding.FaError), e.value
