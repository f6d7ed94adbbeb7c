"""The C ABI on a GPU: invalid buffers are refused before any launch, the
bounded wait gives up with a status instead of hanging, and the context stays
usable afterwards."""

import pytest
import torch

from gpu_helpers import compare, oracle_full, run_cuda, to64
from tiled_online_softmax_03_b200 import binding
from tiled_online_softmax_03_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def tensors(B=1, Hq=2, Hk=1, N=256, d=64, dtype=torch.bfloat16):
    q = torch.randn(B, Hq, N, d, device=DEV).to(dtype)
    k = torch.randn(B, Hk, N, d, device=DEV).to(dtype)
    v = torch.randn(B, Hk, N, d, device=DEV).to(dtype)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, device=DEV)
    return q, k, v, o, lse


def raw(q, k, v, o, lse, B=1, Hq=2, Hk=1, N=256, d=64, lens=None, dtype=1):
    return binding.lib.fa_fwd(q, k, v, o, lse, B, Hq, Hk, N, d, 0.125, 0, lens, None, dtype)


def test_valid_call_returns_ok():
    q, k, v, o, lse = tensors()
    assert raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr()) == 0
    assert binding.device_status() == 0


def test_misaligned_pointer_rejected():
    q, k, v, o, lse = tensors()
    rc = raw(q.data_ptr() + 2, k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr())
    assert rc == binding.FA_ERR_INVALID_ARG and "aligned" in binding.last_error()


def test_host_pointer_rejected():
    q, k, v, o, lse = tensors()
    h = torch.empty(1 << 20, dtype=torch.uint8)
    rc = raw(h.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr())
    assert rc == binding.FA_ERR_INVALID_ARG


def test_buffer_too_small_rejected():
    # a dedicated allocation far smaller than the declared shape
    q, k, v, o, lse = tensors()
    N_big = 1 << 22
    rc = raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), N=N_big)
    assert rc == binding.FA_ERR_INVALID_ARG and "past its allocation" in binding.last_error()


def test_output_overlapping_input_rejected():
    q, k, v, o, lse = tensors()
    rc = raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), q.data_ptr(), lse.data_ptr())
    assert rc == binding.FA_ERR_INVALID_ARG and "overlap" in binding.last_error()


def test_unsupported_head_dim_does_not_fall_back():
    q, k, v, o, lse = tensors(d=64)
    rc = raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), d=48, N=128)
    assert rc == binding.FA_ERR_UNSUPPORTED


def test_binding_checks_dtypes():
    q, k, v, o, lse = tensors()
    with pytest.raises(binding.FaError):
        binding.fa_fwd(q.float(), k.float(), v.float())
    with pytest.raises(binding.FaError):
        binding.fa_fwd(q, k.half(), v)


def test_bounded_wait_gives_up_and_context_survives():
    assert binding.lib.fa_selftest_wait_timeout(200) == 0
    assert binding.device_status() == binding.FA_ERR_DEVICE_TIMEOUT
    assert binding.device_status() == 0  # reading clears it
    w = Workload("after", 1, 2, 1, 300, 64, "bf16", True, seed=2)
    x = make_inputs(w)
    o, lse = run_cuda(x["q"], x["k"], x["v"], True, w.scale, None)
    o_ref, lse_ref = oracle_full(x["q"], x["k"], x["v"], True, w.scale, None)
    compare(to64(o), to64(lse), o_ref, lse_ref, torch.bfloat16)


def test_no_device_memory_allocated_per_call():
    q, k, v, o, lse = tensors(N=1024)
    # one call first, so lazy module loading is not counted
    assert raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), N=1024) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        assert raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                   N=1024) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
