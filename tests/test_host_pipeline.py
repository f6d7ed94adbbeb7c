"""fa_fwd_host (binding: fa_fwd_from_host): the forward on pinned host
buffers, pipelined chunk by chunk (copy in of chunk c + 1, attention of chunk
c, copy out of chunk c − 1 on three streams). Each chunk runs the same kernel
on its slices (whole batches, or runs of K/V heads of one batch), so the
result must equal the device-buffer fa_fwd bit for bit; the oracle comparison
of fa_fwd itself is in test_parity.py.
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


@pytest.mark.parametrize("B,Hq,Hk", [(1, 32, 8), (1, 32, 32), (1, 1, 1), (2, 4, 2), (3, 8, 8),
                                      (4, 32, 8), (4, 32, 1), (32, 16, 16), (33, 2, 1)])
@pytest.mark.parametrize("chunks", [0, 1, 2, 3, 5, 16, 64])
def test_chunk_plan_covers_every_head_once(B, Hq, Hk, chunks):
    """Every (b, K/V head) lands in exactly one chunk; a chunk is one
    contiguous slice (whole batches, or a run of K/V heads of one batch)."""
    from tiled_online_softmax_03_b200.binding import host_chunk_plan
    N, d = 4096, 128
    plan = host_chunk_plan(B, Hq, Hk, N, d, chunks)
    seen = []
    for b0, b1, h0, h1 in plan:
        assert 0 <= b0 < b1 <= B and 0 <= h0 < h1 <= Hk
        if b1 - b0 > 1:
            assert (h0, h1) == (0, Hk), "a multi-batch chunk must hold every head"
        seen += [(b, h) for b in range(b0, b1) for h in range(h0, h1)]
    assert seen == [(b, h) for b in range(B) for h in range(Hk)]  # in order, once each
    if chunks:
        if B >= chunks:
            assert len(plan) == chunks
        else:
            assert len(plan) == B * min(Hk, -(-chunks // B))
    else:  # default: about 16 MB of inputs per chunk, at most 16 chunks
        mb = 2 * B * N * d * (Hq + 2 * Hk) / 2 ** 20
        want = max(1, min(16, int(mb // 16)))
        assert len(plan) == (want if B >= want else B * min(Hk, -(-want // B)))


def test_chunk_plan_rejects_bad_arguments():
    from tiled_online_softmax_03_b200 import binding
    for args in [(0, 1, 1, 8, 64, 0), (1, 3, 2, 8, 64, 0), (1, 1, 1, 8, 64, -1),
                 (1, 1, 1, 8, 64, 65)]:
        with pytest.raises(binding.FaError):
            binding.host_chunk_plan(*args)


@pytest.mark.gpu
@pytest.mark.parametrize("chunks", [None, 1, 3, 6, 12])
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


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hq,Hk,chunks", [(1, 8, 2, 2), (1, 8, 8, 5), (2, 8, 4, 4), (1, 4, 4, 3)])
def test_head_chunks_equal_device_call(B, Hq, Hk, chunks):
    """Chunks that cut a batch into runs of K/V heads (B below the chunk count)."""
    from tiled_online_softmax_03_b200 import binding
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    w, x, L = _host_inputs(B, Hq, Hk, 700, 128, "bf16", True, [650, 333][:B], seed=3 + B + Hk)
    dev = torch.device("cuda:0")
    o_ref, l_ref = binding.fa_fwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), causal=True,
                                  key_pad_lens=L.to(dev))
    hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
    assert len(binding.host_chunk_plan(B, Hq, Hk, 700, 128, chunks)) > B
    o, lse = binding.fa_fwd_from_host(hq, hk, hv, causal=True, key_pad_lens=L.pin_memory(),
                                      chunks=chunks)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    assert torch.equal(o, o_ref.cpu()) and torch.equal(lse, l_ref.cpu())


@pytest.mark.gpu
@pytest.mark.parametrize("as_handle", [False, True])
def test_side_stream_with_owned_buffers(as_handle):
    """Two calls on a side stream (a torch stream, or its raw handle) with the
    device buffers allocated by the call, and allocations on the current
    stream in between: both results equal fa_fwd bit for bit."""
    from tiled_online_softmax_03_b200 import binding
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dev = torch.device("cuda:0")
    side = torch.cuda.Stream(dev)
    B, Hq, Hk, N, d = 2, 8, 2, 1024, 128
    results = []
    for seed in (21, 22):
        w, x, _ = _host_inputs(B, Hq, Hk, N, d, "bf16", True, seed=seed)
        hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
        o, lse = binding.fa_fwd_from_host(hq, hk, hv, causal=True, device=dev,
                                          stream=side.cuda_stream if as_handle else side)
        junk = [torch.full((1 << 20,), 3.0, device=dev) for _ in range(8)]  # reuse pressure
        del junk
        results.append((x, o, lse))
    side.synchronize()
    assert binding.device_status() == 0
    for x, o, lse in results:
        o_ref, l_ref = binding.fa_fwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), causal=True)
        assert torch.equal(o, o_ref.cpu()) and torch.equal(lse, l_ref.cpu())


@pytest.mark.gpu
def test_stream_on_another_device_or_pageable_memory_is_refused():
    from tiled_online_softmax_03_b200 import binding
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B, Hq, Hk, N, d = 1, 2, 1, 128, 64
    w, x, _ = _host_inputs(B, Hq, Hk, N, d, "bf16", False, seed=2)
    hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
    if torch.cuda.device_count() > 1:
        with pytest.raises(binding.FaError, match="stream"):
            binding.fa_fwd_from_host(hq, hk, hv, device=torch.device("cuda:0"),
                                     stream=torch.cuda.Stream(torch.device("cuda:1")))
    # the C call itself refuses pageable host memory
    dev = torch.device("cuda:0")
    bufs = [torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (hq, hk, hv, hq)]
    lse_d = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    out = torch.empty(hq.shape, dtype=hq.dtype)  # not pinned
    rc = binding.lib.fa_fwd_host(hq.data_ptr(), hk.data_ptr(), hv.data_ptr(), out.data_ptr(), None,
                                 B, Hq, Hk, N, d, 0.125, 0, None, bufs[0].data_ptr(),
                                 bufs[1].data_ptr(), bufs[2].data_ptr(), bufs[3].data_ptr(), None,
                                 None, 0, None, binding.FA_BF16)
    assert rc == binding.FA_ERR_INVALID_ARG and "pinned" in binding.last_error()


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
