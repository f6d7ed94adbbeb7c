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


# ----------------------------------------------------- split-KV decomposition

SPLIT_SHAPES = [(1, 1, 1, 128, 0), (2, 4, 2, 300, 1), (2, 3, 1, 513, 0), (1, 8, 1, 2048, 1),
                (1, 6, 2, 1000, 1), (3, 5, 5, 129, 1), (1, 2, 2, 1, 0)]


def needed_tiles(N, causal, mb, key_len):
    end = min(key_len, (mb + 1) * 128) if causal else key_len
    return (end + 127) // 128 if end > 0 else 0


@pytest.mark.parametrize("B,Hq,Hk,N,causal", SPLIT_SHAPES)
@pytest.mark.parametrize("splits", [1, 2, 3, 4, 7, 16])
def test_split_ranges_partition_each_tiles_keys(B, Hq, Hk, N, causal, splits):
    """Across the splits of a tile pair, each Q tile visits every K/V tile it
    needs exactly once, and a split's tiles are one contiguous range."""
    nu = binding.num_units(B, Hq, Hk, N, causal)
    for key_len in sorted({N, max(N // 3, 1), 1, 0}):
        visits = {}
        for u in range(nu * splits):
            r = binding.unit_kv_range(B, Hq, Hk, N, causal, splits, u, key_len)
            assert r[:8] == binding.unit_info(B, Hq, Hk, N, causal, u // splits)
            assert r[8] == u % splits
            j0 = r[9]
            for t, (hq, mb, present, n) in enumerate(((r[2], r[3], r[4], r[10]),
                                                      (r[5], r[6], r[7], r[11]))):
                if not present:
                    continue
                assert n >= j0
                visits.setdefault((r[0], hq, mb), []).extend(range(j0, n))
        assert len(visits) == B * Hq * ((N + 127) // 128)
        for (b, hq, mb), tiles in visits.items():
            assert sorted(tiles) == list(range(needed_tiles(N, causal, mb, key_len)))


def test_split_count_and_workspace_size():
    assert binding.splitkv_workspace_bytes(2, 3, 100, 128, 1) == 0
    assert binding.splitkv_workspace_bytes(2, 3, 100, 128, 17) == 0
    assert binding.splitkv_workspace_bytes(2, 3, 100, 96, 2) == 0
    rows = 2 * 3 * 100 * 4
    rup = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert binding.splitkv_workspace_bytes(2, 3, 100, 128, 4) == rup(rows * 128 * 4) + rup(rows * 4)
    assert binding.splitkv_workspace_bytes(1, 1, 1, 64, 16) == 16 * 64 * 4 + 256
    lib = binding.lib
    for splits in (0, 17, -1):
        assert lib.fa_fwd_splitkv(16, 16, 16, 16, None, 1, 1, 1, 128, 64, 0.1, 0, None, splits,
                                  None, 0, None, 0) == -1
        assert "num_splits" in binding.last_error()
    with pytest.raises(binding.FaError):
        binding.unit_kv_range(1, 1, 1, 128, 0, 2, 2, 128)  # only units 0 and 1 exist
    with pytest.raises(binding.FaError):
        binding.unit_kv_range(1, 1, 1, 128, 0, 2, 0, 129)  # key_len > N


def test_bias_arguments_rejected_before_cuda():
    lib = binding.lib
    # bias_B must be 1 or B, bias_H 1 or Hq; N % 8 != 0 is unsupported; NULL bias rejected
    args = lambda bias, bB, bH, N: (16, 16, 16, bias, bB, bH, 16, None, 2, 4, 2, N, 64, 0.1, 0,  # noqa: E731
                                    None, None, 1)
    assert lib.fa_fwd_bias(*args(16, 3, 1, 64)) == -1 and "batch" in binding.last_error()
    assert lib.fa_fwd_bias(*args(16, 1, 2, 64)) == -1 and "head" in binding.last_error()
    assert lib.fa_fwd_bias(*args(16, 2, 4, 60)) == -2 and "N % 8" in binding.last_error()
    assert lib.fa_fwd_bias(*args(None, 1, 1, 64)) == -1 and "NULL" in binding.last_error()


def test_backward_arguments_rejected_before_cuda():
    lib = binding.lib
    args = lambda d, N, Hq=2, Hk=1, scale=0.1, causal=0, ws=1 << 30: (  # noqa: E731
        16, 16, 16, 16, 16, 16, 16, 16, 16, 1, Hq, Hk, N, d, scale, causal, None, 16, ws, None, 1)
    assert lib.fa_bwd(*args(96, 128)) == -2 and "head dim" in binding.last_error()
    assert lib.fa_bwd(*args(128, 128, Hq=3, Hk=2)) == -1 and "multiple" in binding.last_error()
    assert lib.fa_bwd(*args(128, 128, scale=float("nan"))) == -1
    assert lib.fa_bwd(*args(128, 128, causal=2)) == -1
    assert lib.fa_bwd(*args(128, 128, ws=0)) == -1 and "workspace" in binding.last_error()
    nulls = (None,) + (16,) * 8 + (1, 2, 1, 128, 128, 0.1, 0, None, 16, 1 << 30, None, 1)
    assert lib.fa_bwd(*nulls) == -1 and "NULL" in binding.last_error()
    need = binding.lib.fa_bwd_workspace_bytes(2, 4, 300, 128)
    npad = 384
    rup = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert need == rup(8 * 300 * 128 * 4) + 2 * rup(8 * npad * 4)
    assert binding.lib.fa_bwd_workspace_bytes(2, 4, 300, 80) == 0


def test_fp8_arguments_rejected_before_cuda():
    lib = binding.lib
    args = lambda d, N, qs=1.0, ws=1 << 30: (16, 16, 16, qs, 1.0, 1.0, 16, None, 1, 2, 1, N, d,  # noqa: E731
                                             0.1, 0, None, 16, ws, None)
    assert lib.fa_fwd_fp8(*args(64, 128)) == -2 and "head dim" in binding.last_error()
    assert lib.fa_fwd_fp8(*args(128, 100)) == -2 and "N % 16" in binding.last_error()
    assert lib.fa_fwd_fp8(*args(128, 128, qs=0.0)) == -1 and "descale" in binding.last_error()
    assert lib.fa_fwd_fp8(*args(128, 128, qs=float("inf"))) == -1
    assert lib.fa_fwd_fp8(*args(128, 128, ws=0)) == -1 and "workspace" in binding.last_error()
    assert binding.lib.fa_fwd_fp8_workspace_bytes(1, 2, 4096, 128) == 2 * 4096 * 128
    assert binding.lib.fa_fwd_fp8_workspace_bytes(1, 2, 4096, 64) == 0


# ------------------------------------------------ head-grouped causal order

GROUP_SHAPES = [(4, 32, 8, 8192, 1, 148), (1, 32, 32, 4096, 1, 148), (4, 32, 1, 8192, 1, 148),
                (1, 16, 16, 32768, 1, 148), (2, 4, 2, 300, 1, 148), (32, 16, 16, 512, 0, 148),
                (3, 6, 6, 4096, 1, 16), (5, 4, 2, 2048, 1, 24), (1, 6, 2, 1000, 1, 1)]


L2 = 126 << 20  # B200


def test_group_policy_on_the_workloads():
    # 8K GQA: 32 (b, hk) heads of 4 MiB K+V on 148 CTAs -> 12 heads (48 MiB) per group -> 3 groups
    assert binding.unit_groups(4, 32, 8, 8192, 128, 1, 148, L2) == 3
    # the 32K workload: 8 (b, hk) heads, ~18 CTAs on each already: one group
    assert binding.unit_groups(1, 32, 8, 32768, 128, 1, 148, L2) == 0
    # 16 heads at 32K: a group of 12 heads' K+V (192 MiB) would not stay in L2 either: one group
    assert binding.unit_groups(1, 16, 16, 32768, 128, 1, 148, L2) == 0
    # 16 heads at N = 8K fit in half of L2: no groups; 64 of them do not
    assert binding.unit_groups(1, 16, 16, 8192, 128, 1, 148, L2) == 0
    assert binding.unit_groups(4, 16, 16, 8192, 128, 1, 148, L2) == 3
    # enough CTAs per head already, or too few units, or not causal: one group
    assert binding.unit_groups(4, 32, 1, 8192, 128, 1, 148, L2) == 0
    assert binding.unit_groups(1, 32, 32, 4096, 128, 1, 148, L2) == 0
    assert binding.unit_groups(32, 16, 16, 512, 64, 0, 148, L2) == 0
    assert binding.unit_groups(2, 4, 2, 300, 128, 1, 148, L2) == 0
    with pytest.raises(binding.FaError):
        binding.unit_groups(1, 3, 2, 128, 128, 1, 148, L2)


@pytest.mark.parametrize("B,Hq,Hk,N,causal,grid", GROUP_SHAPES)
def test_grouped_order_is_a_permutation_heaviest_first_per_group(B, Hq, Hk, N, causal, grid):
    heads = B * Hk
    nu = binding.num_units(B, Hq, Hk, N, causal)
    np_ = nu // heads
    ngs = {binding.unit_groups(B, Hq, Hk, N, 128, causal, grid, L2)} | ({2, min(5, heads)} if causal else set())
    for ng in sorted(ngs):
        plain = {tuple(binding.unit_info(B, Hq, Hk, N, causal, u)) for u in range(nu)}
        got = [binding.unit_kv_range_grouped(B, Hq, Hk, N, causal, 1, ng, u, N) for u in range(nu)]
        assert {tuple(r[:8]) for r in got} == plain  # same units, each once
        if ng < 2 or not causal:
            assert got == [binding.unit_kv_range(B, Hq, Hk, N, causal, 1, u, N) for u in range(nu)]
            continue
        # contiguous groups of near-equal head counts, the larger groups first
        base, rem = divmod(heads, ng)
        u = 0
        bhk_next = 0
        for g in range(ng):
            gh = base + (g < rem)
            chunk = got[u:u + gh * np_]
            members = sorted({r[0] * Hk + r[1] for r in chunk})
            assert members == list(range(bhk_next, bhk_next + gh))
            work = [max(r[3], r[6] if r[7] else 0) for r in chunk]
            assert work == sorted(work, reverse=True)  # heaviest first within the group
            u += gh * np_
            bhk_next += gh
        assert u == nu


def test_grouped_ranges_match_the_plain_ones_per_unit():
    B, Hq, Hk, N = 2, 6, 3, 1000
    nu = binding.num_units(B, Hq, Hk, N, 1)
    for splits in (1, 3):
        plain = {}
        for u in range(nu * splits):
            r = binding.unit_kv_range(B, Hq, Hk, N, 1, splits, u, 700)
            plain[(r[0], r[1], r[2], r[3], r[8])] = r
        for u in range(nu * splits):
            r = binding.unit_kv_range_grouped(B, Hq, Hk, N, 1, splits, 4, u, 700)
            assert plain.pop((r[0], r[1], r[2], r[3], r[8])) == r
        assert not plain
    with pytest.raises(binding.FaError):
        binding.unit_kv_range_grouped(B, Hq, Hk, N, 1, 1, B * Hk + 1, 0, N)


@pytest.mark.parametrize("B,Hq,Hk,N,grid,groups,splits",
                         [(4, 32, 8, 8192, 148, 3, 1), (4, 32, 8, 8192, 148, 2, 1),
                          (1, 16, 16, 32768, 148, 2, 1), (3, 6, 6, 4096, 16, 4, 1),
                          (5, 4, 2, 2048, 24, 3, 2), (2, 4, 2, 300, 7, 4, 3), (1, 6, 2, 1000, 1, 2, 1)])
def test_grouped_assignment_partitions_each_group_in_turn(B, Hq, Hk, N, grid, groups, splits):
    nu = binding.num_units(B, Hq, Hk, N, 1) * splits
    heads = B * Hk
    per_head = nu // heads
    base, rem = divmod(heads, groups)
    bounds = []  # first unit of each group
    x = 0
    for g in range(groups):
        bounds.append(x)
        x += (base + (g < rem)) * per_head
    grid = min(grid, nu)
    got = []
    for cta in range(grid):
        seq = []
        it = 0
        while True:
            u = binding.unit_for_grouped(B, Hq, Hk, N, 1, splits, groups, cta, it, grid)
            if u >= nu:
                break
            seq.append(u)
            it += 1
        gs = [max(i for i, b in enumerate(bounds) if b <= u) for u in seq]
        assert gs == sorted(gs)  # groups in turn
        assert seq == sorted(seq)  # and in list order (heaviest first) inside each group
        got.extend(seq)
    assert sorted(got) == list(range(nu))
    # each group is dealt out by itself: its units go to the CTAs as evenly as possible
    for g in range(groups):
        lo = bounds[g]
        hi = bounds[g + 1] if g + 1 < groups else nu
        counts = {}
        for cta in range(grid):
            it = 0
            while True:
                u = binding.unit_for_grouped(B, Hq, Hk, N, 1, splits, groups, cta, it, grid)
                if u >= nu:
                    break
                if lo <= u < hi:
                    counts[cta] = counts.get(cta, 0) + 1
                it += 1
        c = [counts.get(cta, 0) for cta in range(grid)]
        assert max(c) - min(c) <= 1 and sum(c) == hi - lo
