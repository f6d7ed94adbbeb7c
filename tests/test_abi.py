"""The C ABI without a GPU: the library loads, exports what include/fa.h
declares, rejects bad arguments before touching CUDA, and its work
decomposition covers every Q tile exactly once in the documented order."""

import ctypes
import os
import re

import pytest

from tiled_online_softmax_03_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "fa.h"), encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert "fa_fwd" in names and len(names) >= 8
    lib = ctypes.CDLL(binding.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/fa.h but not exported"


def test_version():
    assert binding.lib.fa_version() >= 100


def call(*args):
    return binding.lib.fa_fwd(*args)


def test_null_pointers_rejected():
    assert call(None, 1, 1, 1, None, 1, 1, 1, 128, 64, 0.1, 0, None, None, 0) == -1
    assert "NULL" in binding.last_error()
    assert call(16, 16, 16, None, None, 1, 1, 1, 128, 64, 0.1, 0, None, None, 0) == -1


@pytest.mark.parametrize("B,Hq,Hk,N", [(0, 1, 1, 8), (1, 0, 1, 8), (1, 1, 0, 8), (1, 1, 1, 0),
                                       (1, 3, 2, 8), (-1, 1, 1, 8)])
def test_bad_shapes_rejected(B, Hq, Hk, N):
    assert call(16, 16, 16, 16, None, B, Hq, Hk, N, 64, 0.1, 0, None, None, 0) == -1


@pytest.mark.parametrize("d", [0, 16, 32, 48, 80, 96, 256])
def test_head_dims_other_than_64_128_unsupported(d):
    assert call(16, 16, 16, 16, None, 1, 1, 1, 8, d, 0.1, 0, None, None, 0) == -2
    assert "head dim" in binding.last_error()


def test_bad_dtype_scale_causal():
    assert call(16, 16, 16, 16, None, 1, 1, 1, 8, 64, 0.1, 0, None, None, 7) == -2
    assert call(16, 16, 16, 16, None, 1, 1, 1, 8, 64, float("nan"), 0, None, None, 0) == -1
    assert call(16, 16, 16, 16, None, 1, 1, 1, 8, 64, float("inf"), 0, None, None, 0) == -1
    assert call(16, 16, 16, 16, None, 1, 1, 1, 8, 64, 0.1, 2, None, None, 0) == -1


def test_wait_timeout_setter():
    assert binding.lib.fa_set_wait_timeout_ms(0) == -1
    assert binding.lib.fa_set_wait_timeout_ms(600001) == -1
    assert binding.lib.fa_set_wait_timeout_ms(4000) == 0


# ------------------------------------------------------------ the schedule

SHAPES = [(1, 1, 1, 128, 0), (1, 1, 1, 1, 1), (2, 4, 2, 300, 1), (2, 3, 1, 513, 0),
          (4, 32, 8, 8192, 1), (4, 32, 1, 8192, 1), (1, 32, 32, 4096, 1), (32, 16, 16, 512, 0),
          (1, 6, 2, 1000, 1), (3, 5, 5, 129, 1)]


@pytest.mark.parametrize("B,Hq,Hk,N,causal", SHAPES)
def test_units_cover_every_q_tile_once(B, Hq, Hk, N, causal):
    nu = binding.num_units(B, Hq, Hk, N, causal)
    nm = (N + 127) // 128
    G = Hq // Hk
    assert nu == B * Hk * ((G * nm + 1) // 2)
    seen = set()
    for u in range(nu):
        b, hk, hq0, mb0, p0, hq1, mb1, p1 = binding.unit_info(B, Hq, Hk, N, causal, u)
        assert 0 <= b < B and 0 <= hk < Hk and p0 == 1
        for hq, mb, present in ((hq0, mb0, p0), (hq1, mb1, p1)):
            if not present:
                continue
            assert hq // G == hk, "both tiles of a unit must read the unit's K/V head"
            assert 0 <= mb < nm
            assert (b, hq, mb) not in seen
            seen.add((b, hq, mb))
    assert len(seen) == B * Hq * nm


@pytest.mark.parametrize("B,Hq,Hk,N,causal", [s for s in SHAPES if s[4]])
def test_causal_units_are_heaviest_first(B, Hq, Hk, N, causal):
    nu = binding.num_units(B, Hq, Hk, N, causal)
    last = None
    for u in range(nu):
        info = binding.unit_info(B, Hq, Hk, N, causal, u)
        work = max(info[3], info[6] if info[7] else 0)
        if last is not None:
            assert work <= last
        last = work


@pytest.mark.parametrize("grid,units", [(148, 4096), (148, 1), (148, 1024), (7, 100), (1, 5)])
def test_serpentine_assignment_is_a_partition(grid, units):
    got = []
    for cta in range(min(grid, units)):
        it = 0
        while True:
            u = binding.unit_for(cta, it, min(grid, units))
            if u >= units:
                break
            got.append(u)
            it += 1
    assert sorted(got) == list(range(units))


def test_unit_info_rejects_bad_index():
    with pytest.raises(binding.FaError):
        binding.unit_info(1, 1, 1, 128, 0, 5)
