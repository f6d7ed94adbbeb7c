"""The FMA-pipe exponential the softmax uses for part of its 2^x values.

Host side: the coefficients in the kernel are those the committed Remez fit
produces, and a float32 model of the kernel's arithmetic stays within the
fit's bound. Device side: the kernel's own function against the exact 2^x
and against ex2.approx (CUDA's hardware approximation).
"""

import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tiled_online_softmax_03_b200", "csrc")
BOUND = 1e-4  # relative; the largest 16-bit rounding P gets next is 4.9e-4 (fp16)


def fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def kernel_coefficients():
    src = open(os.path.join(CSRC, "fa_fwd_sm100.cu"), encoding="utf-8").read()
    vals = dict(re.findall(r"constexpr float EXP2_C(\d) = ([0-9.e+-]+)f;", src))
    return np.array([float(vals[str(i)]) for i in range(4)], dtype=np.float32)


def test_kernel_coefficients_are_the_fit():
    m = fit_module()
    fitted = m.remez_relative().astype(np.float32)
    assert np.array_equal(kernel_coefficients(), fitted)


def test_float32_model_error_bound():
    m = fit_module()
    c = kernel_coefficients()
    x = np.concatenate([np.linspace(-125.9, 9.0, 1000001), np.arange(-125, 10)]).astype(np.float32)
    y = m.exp2_emulated_f32(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < BOUND
    # below the clamp the result is at most 2^-125 (negligible next to P's maximum of 1)
    tiny = m.exp2_emulated_f32(np.array([-126.5, -200.0, -1e30], dtype=np.float32), c)
    assert np.all(tiny >= 0) and np.all(tiny <= 2.0 ** -125)


def test_remez_error_levels_out():
    """The fit equioscillates: a degree-3 polynomial cannot do much better."""
    m = fit_module()
    c = m.remez_relative()
    g = np.linspace(-0.5, 0.5, 200001)
    err = np.polyval(c[::-1], g) / 2.0 ** g - 1.0
    assert abs(err.max() + err.min()) < 0.05 * err.max()
    assert err.max() < 8e-5


@pytest.mark.gpu
def test_device_exp2_against_exact_and_mufu():
    import ctypes

    import torch

    from tiled_online_softmax_03_b200 import binding
    assert torch.cuda.is_available()
    x = torch.cat([torch.linspace(-125.9, 9.0, 1 << 20), torch.arange(-125, 10).float(),
                   torch.tensor([-126.5, -300.0])]).cuda()
    yf = torch.empty_like(x)
    ym = torch.empty_like(x)
    binding.lib.fa_selftest_exp2.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    assert binding.lib.fa_selftest_exp2(x.data_ptr(), yf.data_ptr(), ym.data_ptr(), x.numel()) == 0
    xd = x.double().cpu().numpy()
    yf = yf.double().cpu().numpy()
    ym = ym.double().cpu().numpy()
    ok = xd >= -125.9
    exact = np.exp2(xd[ok])
    assert np.max(np.abs(yf[ok] / exact - 1)) < BOUND
    assert np.max(np.abs(yf[ok] / ym[ok] - 1)) < BOUND + 1e-6
    assert np.all(yf[~ok] <= 2.0 ** -125) and np.all(yf[~ok] >= 0)
    # matches the float32 host model (the device fuses each multiply-add: within 2 ulp)
    m = fit_module()
    host = m.exp2_emulated_f32(xd.astype(np.float32), kernel_coefficients()).astype(np.float64)
    assert np.max(np.abs(yf[ok] / host[ok] - 1)) < 2.5e-7
