"""Guard bands around every buffer the kernels write (compute-sanitizer is not
available here): each output and workspace is a slice in the middle of a larger
allocation whose head and tail are filled with a sentinel byte pattern; after
the call (and a device sync) the bands must be unchanged and the outputs
finite. Ragged N and key padding put rows and keys past every tile boundary.
"""

import pytest
import torch

from tiled_online_softmax_03_b200.inputs import Workload, make_bias, make_inputs

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side
SENTINEL = 0xA5


@pytest.fixture(autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


class Guarded:
    """A tensor view with sentinel bands of GUARD bytes before and after it."""

    def __init__(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + nbytes + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape)
        self.nbytes = nbytes

    def check(self):
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.nbytes:]
        assert bool((head == SENTINEL).all()), "write before the buffer"
        assert bool((tail == SENTINEL).all()), "write past the buffer"


def inputs(B, Hq, Hk, N, d, dtype, causal, lens=None, seed=0):
    w = Workload("g", B, Hq, Hk, N, d, dtype, causal, seed=seed)
    x = make_inputs(w)
    dev = torch.device("cuda:0")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    L = torch.tensor(lens, dtype=torch.int32, device=dev) if lens is not None else None
    return w, q, k, v, L


@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "fp16")])
@pytest.mark.parametrize("causal", [False, True])
def test_forward_writes_stay_in_bounds(d, dtype, causal):
    from tiled_online_softmax_03_b200 import binding
    w, q, k, v, L = inputs(3, 4, 2, 333, d, dtype, causal, lens=[333, 0, 130], seed=d)
    o = Guarded(q.shape, q.dtype)
    lse = Guarded((3, 4, 333), torch.float32)
    binding.fa_fwd(q, k, v, causal=causal, key_pad_lens=L, out=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o.check()
    lse.check()
    assert torch.isfinite(o.t).all()


def test_splitkv_and_static_writes_stay_in_bounds():
    from tiled_online_softmax_03_b200 import binding
    w, q, k, v, L = inputs(2, 4, 2, 650, 128, "bf16", True, lens=[650, 200], seed=3)
    need = binding.splitkv_workspace_bytes(2, 4, 650, 128, 3)
    ws = Guarded((need,), torch.uint8)
    o = Guarded(q.shape, q.dtype)
    lse = Guarded((2, 4, 650), torch.float32)
    binding.fa_fwd_splitkv(q, k, v, 3, causal=True, key_pad_lens=L, out=o.t, lse=lse.t,
                           workspace=ws.t)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    for g in (ws, o, lse):
        g.check()
    o2 = Guarded(q.shape, q.dtype)
    binding.fa_fwd_splitkv_static(q, k, v, 3, causal=True, key_pad_lens=L, out=o2.t)
    torch.cuda.synchronize()
    o2.check()
    assert torch.equal(o.t, o2.t)


def test_bias_writes_stay_in_bounds():
    from tiled_online_softmax_03_b200 import binding
    w, q, k, v, L = inputs(2, 2, 1, 264, 128, "bf16", False, lens=[264, 100], seed=4)
    bias = make_bias(w, 1, 2, device="cuda")
    o = Guarded(q.shape, q.dtype)
    lse = Guarded((2, 2, 264), torch.float32)
    binding.fa_fwd_bias(q, k, v, bias, key_pad_lens=L, out=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o.check()
    lse.check()


@pytest.mark.parametrize("d", [64, 128])
def test_backward_writes_stay_in_bounds(d):
    from tiled_online_softmax_03_b200 import binding
    w, q, k, v, L = inputs(2, 4, 2, 300, d, "bf16", True, lens=[300, 150], seed=5)
    o, lse = binding.fa_fwd(q, k, v, causal=True, key_pad_lens=L)
    dout = torch.randn_like(q)
    dq = Guarded(q.shape, q.dtype)
    dk = Guarded(k.shape, k.dtype)
    dv = Guarded(v.shape, v.dtype)
    ws = Guarded((binding.lib.fa_bwd_workspace_bytes(2, 4, 300, d),), torch.uint8)
    binding.fa_bwd(q, k, v, o, lse, dout, causal=True, key_pad_lens=L, dq=dq.t, dk=dk.t,
                   dv=dv.t, workspace=ws.t)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    for g in (dq, dk, dv, ws):
        g.check()
    assert torch.isfinite(dq.t).all() and torch.isfinite(dk.t).all() and torch.isfinite(dv.t).all()


def test_fp8_writes_stay_in_bounds():
    from tiled_online_softmax_03_b200 import binding
    fp8 = torch.float8_e4m3fn
    g = torch.Generator().manual_seed(6)
    q, k, v = (torch.randn(s, generator=g).to(fp8).cuda() for s in
               [(2, 4, 272, 128), (2, 2, 272, 128), (2, 2, 272, 128)])
    o = Guarded((2, 4, 272, 128), torch.bfloat16)
    lse = Guarded((2, 4, 272), torch.float32)
    ws = Guarded((binding.lib.fa_fwd_fp8_workspace_bytes(2, 2, 272, 128),), torch.uint8)
    binding.fa_fwd_fp8(q, k, v, 1.0, 1.0, 1.0, causal=True, out=o.t, lse=lse.t, workspace=ws.t)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    for gd in (o, lse, ws):
        gd.check()
    assert torch.isfinite(o.t).all()
