"""Pins for the float64 oracle, each against something other than the orc.

Sources of the pins: closed forms, invariants of softmax attention, a library
routine (torch's float64 math SDPA), brute force over tiny inputs in exact
summation, and the pages' own claims (the online recurrence of the MCU page's
§二 equals the two-pass softmax exactly; causal row 0 sees only key 0; GQA
shares one K/V head across a group of query heads).
"""

import itertools
import json
import math
import os

import numpy as np
import torch


RNG = np.random.default_rng(1234)


def rand(*shape, rng=RNG):
    return rng.standard_normal(shape)


def brute_force(q, k, v, scale, causal, lens, key_lo=0, key_hi=None, bias=None):
    """Scalar loops with math.fsum: one row at a time, no vectorised code.

    Only keys key_lo <= j < key_hi take part (all keys by default); bias, if
    given, is a full [B, Hq, N, N] array added to each score."""
    B, Hq, N, d = q.shape
    Hk = k.shape[1]
    G = Hq // Hk
    o = np.zeros((B, Hq, N, v.shape[3]))
    lse = np.full((B, Hq, N), -math.inf)
    for b in range(B):
        L = N if lens is None else min(max(int(lens[b]), 0), N)
        for h in range(Hq):
            kh = h // G
            for i in range(N):
                hi = N if key_hi is None else key_hi
                keys = [j for j in range(key_lo, hi) if j < L and (not causal or j <= i)]
                if not keys:
                    continue
                s = {j: scale * math.fsum(q[b, h, i, c] * k[b, kh, j, c] for c in range(d))
                     + (0.0 if bias is None else bias[b, h, i, j]) for j in keys}
                mx = max(s.values())
                w = {j: math.exp(s[j] - mx) for j in keys}
                tot = math.fsum(w.values())
                for c in range(v.shape[3]):
                    o[b, h, i, c] = math.fsum(w[j] * v[b, kh, j, c] for j in keys) / tot
                lse[b, h, i] = mx + math.log(tot)
    return o, lse


def close(a, b, tol=1e-12):
    a, b = np.asarray(a), np.asarray(b)
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin)
    assert np.array_equal(a[~fin], b[~fin])
    if fin.any():
        assert np.max(np.abs(a[fin] - b[fin])) <= tol * max(1.0, np.max(np.abs(b[fin])))


# ---------------------------------------------------------------- brute force

def pin_matches_scalar_brute_force(orc):
    q, k, v = rand(2, 4, 6, 3), rand(2, 2, 6, 3), rand(2, 2, 6, 2)
    for causal, lens in itertools.product([False, True], [None, [3, 0]]):
        o, lse = orc.attention(q, k, v, 0.7, causal, lens)
        ob, lseb = brute_force(q, k, v, 0.7, causal, lens)
        close(o, ob)
        close(lse, lseb)


# ------------------------------------------------------------ library routine

def pin_matches_torch_math_sdpa(orc):
    for causal, G in itertools.product([False, True], [1, 2, 4]):
        _sdpa_case(orc, causal, G)


def _sdpa_case(orc, causal, G):
    B, Hk, N, d = 2, 2, 37, 16
    Hq = Hk * G
    q, k, v = rand(B, Hq, N, d), rand(B, Hk, N, d), rand(B, Hk, N, d)
    lens = [37, 20]
    scale = 0.3
    o, _ = orc.attention(q, k, v, scale, causal, lens)
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    mask = torch.stack([(j < L) & ((j <= i) if causal else torch.ones_like(j <= i))
                        for L in lens])[:, None]
    kt = torch.from_numpy(k).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(G, dim=1)
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), kt, vt, attn_mask=mask, scale=scale).numpy()
    close(o, ref, 1e-12)


# ------------------------------------------------- recurrence == two-pass ([MCU] §二)

def pin_online_recurrence_equals_two_pass_all_tilings(orc):
    for fn in (orc.online_attention_flowchart, orc.online_attention_equations):
        _all_tilings(orc, fn)


def _all_tilings(orc, fn):
    rng = np.random.default_rng(7)
    N, d = 7, 3
    q, k, v = rng.standard_normal((1, 2, N, d)), rng.standard_normal((1, 1, N, d)), \
        rng.standard_normal((1, 1, N, 2))
    for causal, lens in [(False, None), (True, None), (False, [4]), (True, [5]), (False, [0])]:
        ref_o, ref_l = orc.attention(q, k, v, 1.3, causal, lens)
        for tr, tc in itertools.product(range(1, N + 1), repeat=2):
            o, l = fn(q, k, v, 1.3, causal, lens, tile_r=tr, tile_c=tc)
            close(o, ref_o, 1e-12)
            close(l, ref_l, 1e-12)


def pin_online_recurrence_adversarial_scores(orc):
    """Increasing, decreasing and ±30-spread scores force every rescale branch."""
    for fn in (orc.online_attention_flowchart, orc.online_attention_equations):
        _adversarial(orc, fn)


def _adversarial(orc, fn):
    N = 9
    v = RNG.standard_normal((1, 1, N, 3))
    k = np.zeros((1, 1, N, 1))
    q = np.ones((1, 1, N, 1))
    for keys in [np.arange(N) * 4.0, -np.arange(N) * 4.0, np.array([30, -30] * 4 + [0.0])]:
        k[0, 0, :, 0] = keys
        ref_o, ref_l = orc.attention(q, k, v, 1.0, False, None)
        for tc in range(1, N + 1):
            o, l = fn(q, k, v, 1.0, False, None, tile_r=N, tile_c=tc)
            close(o, ref_o, 1e-12)
            close(l, ref_l, 1e-12)


# ------------------------------------------------------------------ invariants

def pin_softmax_rows_sum_to_one_and_are_nonnegative(orc):
    q, k = rand(5, 8), rand(9, 8)
    for causal, L in [(False, 9), (True, 9), (False, 4), (True, 2)]:
        ok = orc.allowed_keys(np.arange(5), 9, causal, L)
        p, m, l = orc.two_pass_softmax(orc.scores(q, k, 0.5, ok))
        w = p / l[:, None]
        assert np.all(w >= 0)
        assert np.all(w[~ok] == 0)
        assert np.max(np.abs(w.sum(axis=1) - 1.0)) < 1e-12
        assert np.max(p) == 1.0  # the row max contributes exp(0)


def pin_uniform_v_returns_v(orc):
    q, k = rand(1, 3, 11, 4) * 5, rand(1, 3, 11, 4) * 5
    c = rand(4)
    v = np.broadcast_to(c, (1, 3, 11, 4)).copy()
    for causal in (False, True):
        o, _ = orc.attention(q, k, v, 1.0, causal, [7])
        close(o, np.broadcast_to(c, o.shape), 1e-13)


def pin_one_hot_score_selects_v_row(orc):
    """Row i scores key t(i) at 60 and every other key at 0: O_i = V_t(i) within e^-60."""
    N = 10
    v = rand(1, 1, N, 5)
    target = RNG.permutation(N)
    k = np.eye(N)[None, None] * 60.0
    q = np.zeros((1, 1, N, N))
    q[0, 0, np.arange(N), target] = 1.0
    o, lse = orc.attention(q, k, v, 1.0, False, None)
    assert np.max(np.abs(o[0, 0] - v[0, 0, target])) < 1e-14
    assert np.max(np.abs(lse[0, 0] - 60.0)) < 1e-12


def pin_single_allowed_key_is_exact(orc):
    """Key padding to one key: O_i = V_0 and LSE_i = s_i0, exactly."""
    q, k, v = rand(1, 2, 8, 4), rand(1, 1, 8, 4), rand(1, 1, 8, 4)
    o, lse = orc.attention(q, k, v, 0.9, False, [1])
    assert np.array_equal(o[0], np.broadcast_to(v[0, 0, 0], (2, 8, 4)))
    s0 = 0.9 * (q[0, :, :, :] @ k[0, 0, 0])
    assert np.max(np.abs(lse[0] - s0)) < 1e-15 * 8


def pin_causal_row0_is_v0_and_future_keys_do_not_matter(orc):
    q, k, v = rand(1, 1, 12, 4), rand(1, 1, 12, 4), rand(1, 1, 12, 3)
    o, lse = orc.attention(q, k, v, 0.8, True, None)
    assert np.array_equal(o[0, 0, 0], v[0, 0, 0])
    assert lse[0, 0, 0] == 0.8 * (q[0, 0, 0] @ k[0, 0, 0])
    for i in range(12):
        k2, v2 = k.copy(), v.copy()
        k2[0, 0, i + 1:] = rand(12 - i - 1, 4) * 9
        v2[0, 0, i + 1:] = rand(12 - i - 1, 3) * 9
        o2, lse2 = orc.attention(q, k2, v2, 0.8, True, None)
        assert np.array_equal(o2[0, 0, : i + 1], o[0, 0, : i + 1])
        assert np.array_equal(lse2[0, 0, : i + 1], lse[0, 0, : i + 1])


def pin_scale_zero_closed_form(orc):
    """scale = 0: O_i is the mean of the allowed V rows and LSE_i = ln(#allowed)."""
    N = 9
    q, k, v = rand(1, 1, N, 4), rand(1, 1, N, 4), rand(1, 1, N, 3)
    for causal, L in [(False, N), (True, N), (False, 5), (True, 4)]:
        o, lse = orc.attention(q, k, v, 0.0, causal, [L])
        for i in range(N):
            n_ok = min(L, i + 1) if causal else L
            assert np.max(np.abs(o[0, 0, i] - v[0, 0, :n_ok].mean(axis=0))) < 1e-14
            assert abs(lse[0, 0, i] - math.log(n_ok)) < 1e-14


def pin_shift_of_row_scores(orc):
    """Adding c to every score of a row leaves O and shifts LSE by c.

    The shift is built into the inputs: an extra feature 1 on every key and c/scale
    on every query, so the oracle sees an ordinary (d+1)-wide problem.
    """
    N, d, scale = 10, 4, 0.6
    q, k, v = rand(1, 2, N, d), rand(1, 1, N, d), rand(1, 1, N, 3)
    c = rand(1, 2, N, 1) * 7
    q2 = np.concatenate([q, c / scale], axis=3)
    k2 = np.concatenate([k, np.ones((1, 1, N, 1))], axis=3)
    for causal, lens in [(False, None), (True, [6])]:
        o, lse = orc.attention(q, k, v, scale, causal, lens)
        o2, lse2 = orc.attention(q2, k2, v, scale, causal, lens)
        close(o2, o, 1e-12)
        close(lse2, lse + c[..., 0], 1e-12)


def pin_permutations(orc):
    N = 11
    q, k, v = rand(1, 1, N, 4), rand(1, 1, N, 4), rand(1, 1, N, 3)
    o, lse = orc.attention(q, k, v, 0.5, False, None)
    perm = RNG.permutation(N)
    o2, lse2 = orc.attention(q, k[:, :, perm], v[:, :, perm], 0.5, False, None)
    close(o2, o, 1e-12)
    close(lse2, lse, 1e-12)
    o3, lse3 = orc.attention(q[:, :, perm], k, v, 0.5, False, None)
    close(o3, o[:, :, perm], 1e-12)
    close(lse3, lse[:, :, perm], 1e-12)


def pin_gqa_equals_mha_on_repeated_kv(orc):
    for Hq, Hk in [(4, 2), (8, 2), (6, 1), (4, 4)]:
        _gqa_case(orc, Hq, Hk)


def _gqa_case(orc, Hq, Hk):
    q, k, v = rand(2, Hq, 9, 4), rand(2, Hk, 9, 4), rand(2, Hk, 9, 4)
    G = Hq // Hk
    for causal in (False, True):
        o, lse = orc.attention(q, k, v, 0.7, causal, [9, 5])
        o2, lse2 = orc.attention(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1),
                                    0.7, causal, [9, 5])
        close(o, o2, 0)
        close(lse, lse2, 0)


def pin_n_equals_one(orc):
    q, k, v = rand(1, 3, 1, 8), rand(1, 3, 1, 8), rand(1, 3, 1, 8)
    for causal in (False, True):
        o, lse = orc.attention(q, k, v, 0.4, causal, None)
        assert np.array_equal(o, v)
        assert np.max(np.abs(lse[..., 0] - 0.4 * np.einsum("hd,hd->h", q[0, :, 0], k[0, :, 0]))) \
            < 1e-15 * 8


def pin_key_padding_equals_truncated_keys(orc):
    N, L = 12, 7
    q, k, v = rand(1, 2, N, 4), rand(1, 2, N, 4), rand(1, 2, N, 3)
    for causal in (False, True):
        o, lse = orc.attention(q, k, v, 0.5, causal, [L])
        # rows < L with truncated K/V of length L: an independent smaller problem
        o2, lse2 = orc.attention(q[:, :, :L], k[:, :, :L], v[:, :, :L], 0.5, causal, None)
        close(o[:, :, :L], o2, 1e-12)
        close(lse[:, :, :L], lse2, 1e-12)
        if not causal:
            # rows >= L see the same L keys; a row's output is that of the row alone
            for i in range(L, N):
                o3, _ = orc.attention(q[:, :, i:i + 1], k[:, :, :L], v[:, :, :L], 0.5, False, None)
                close(o[:, :, i:i + 1], o3, 1e-12)


def pin_empty_rows(orc):
    q, k, v = rand(2, 2, 5, 4), rand(2, 1, 5, 4), rand(2, 1, 5, 4)
    o, lse = orc.attention(q, k, v, 0.5, True, [0, 5])
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))
    for fn in (orc.online_attention_flowchart, orc.online_attention_equations):
        o2, lse2 = fn(q, k, v, 0.5, True, [0, 5], tile_r=2, tile_c=3)
        close(o2, o, 1e-12)
        close(lse2, lse, 1e-12)


def pin_row_sampling_matches_full(orc):
    q, k, v = rand(2, 4, 33, 8), rand(2, 2, 33, 8), rand(2, 2, 33, 8)
    o, lse = orc.attention(q, k, v, 0.35, True, [33, 17], row_block=5)
    picks = [(0, 0, 0), (1, 3, 32), (1, 1, 16), (0, 2, 20), (1, 2, 20)]
    o2, lse2 = orc.attention_rows(q, k, v, 0.35, True, [33, 17], picks)
    for n, (b, h, i) in enumerate(picks):
        close(o2[n], o[b, h, i], 1e-13)
        close(lse2[n], lse[b, h, i], 1e-13)


def pin_row_block_does_not_change_result(orc):
    q, k, v = rand(1, 2, 40, 8), rand(1, 1, 40, 8), rand(1, 1, 40, 8)
    ref = orc.attention(q, k, v, 0.35, True, None, row_block=1024)
    for rb in (1, 7, 40):
        got = orc.attention(q, k, v, 0.35, True, None, row_block=rb)
        close(got[0], ref[0], 1e-13)
        close(got[1], ref[1], 1e-13)


def pin_large_scores_stay_finite(orc):
    """Scores near ±1000 overflow exp() unless the row max is subtracted first."""
    q, k, v = rand(1, 1, 8, 4), rand(1, 1, 8, 4), rand(1, 1, 8, 3)
    o, lse = orc.attention(q, k, v, 0.5, False, None)
    big = 1000.0 / np.max(np.abs(q))
    c = 900.0
    q2 = np.concatenate([q * 1.0, np.full((1, 1, 8, 1), c / 0.5)], axis=3)
    k2 = np.concatenate([k, np.ones((1, 1, 8, 1))], axis=3)
    o2, lse2 = orc.attention(q2, k2, v, 0.5, False, None)
    close(o2, o, 1e-12)
    close(lse2, lse + c, 1e-12)
    o3, lse3 = orc.attention(q * big, k, v, 0.5, True, None)
    assert np.all(np.isfinite(o3)) and np.all(np.isfinite(lse3))
    for fn in (orc.online_attention_flowchart, orc.online_attention_equations):
        o4, lse4 = fn(q * big, k, v, 0.5, True, None, tile_r=3, tile_c=2)
        close(o4, o3, 1e-12)
        close(lse4, lse3, 1e-12)


def _golden_value(x):
    if isinstance(x, list):
        return [_golden_value(y) for y in x]
    if isinstance(x, str):
        assert x.startswith("ln:")
        return math.log(float(x[3:]))
    return x


def load_golden(name="hand_worked.json"):
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)
    with open(path, encoding="utf-8") as f:
        cases = json.load(f)["cases"]
    out = []
    for c in cases:
        out.append({key: (np.array(_golden_value(c[key]), dtype=np.float64)
                          if key in ("q", "k", "v", "o", "lse") else c[key]) for key in c})
    return out


# ------------------------------------------------ split-KV ([GQA] num_splits)

def pin_key_range_matches_scalar_brute_force(orc):
    q, k, v = rand(1, 2, 7, 3), rand(1, 1, 7, 3), rand(1, 1, 7, 2)
    for causal, lens, lo, hi in itertools.product([False, True], [None, [5]], [0, 2, 3], [3, 6, 7]):
        o, lse = orc.attention_key_range(q, k, v, 0.9, causal, lens, lo, hi)
        ob, lseb = brute_force(q, k, v, 0.9, causal, lens, lo, hi)
        close(o, ob)
        close(lse, lseb)


def pin_split_kv_equals_attention_for_every_cut(orc):
    """Every way of cutting 6 keys into ranges merges back to the full result."""
    rng = np.random.default_rng(11)
    N = 6
    q, k, v = rng.standard_normal((2, 2, N, 3)), rng.standard_normal((2, 1, N, 3)), \
        rng.standard_normal((2, 1, N, 2))
    for causal, lens in [(False, None), (True, None), (False, [4, 0]), (True, [2, 6])]:
        ref_o, ref_l = orc.attention(q, k, v, 1.1, causal, lens)
        for mask in range(1 << (N - 1)):
            cuts = [c for c in range(1, N) if mask >> (c - 1) & 1]
            o, l = orc.split_kv_attention(q, k, v, 1.1, causal, lens, [0] + cuts + [N])
            close(o, ref_o, 1e-12)
            close(l, ref_l, 1e-12)


def pin_merge_closed_form(orc):
    """Two ranges with denominators 1 and 3 at the same max: weights 1/4, 3/4."""
    a, b = np.array([[2.0, -1.0]]), np.array([[6.0, 3.0]])
    o, lse = orc.merge_splits([a, b], [np.array([0.0]), np.array([math.log(3.0)])])
    close(o, [[5.0, 2.0]], 1e-15)
    close(lse, [math.log(4.0)], 1e-15)
    # a range with no allowed key (LSE −inf) has weight 0; no range at all gives 0 / −inf
    o, lse = orc.merge_splits([a, b, b], [np.array([-math.inf]), np.array([1.5]), np.array([-math.inf])])
    close(o, b, 1e-15)
    close(lse, [1.5], 1e-15)
    o, lse = orc.merge_splits([a, b], [np.array([-math.inf]), np.array([-math.inf])])
    close(o, [[0.0, 0.0]])
    close(lse, [-math.inf])


def pin_merge_large_lse_stays_finite(orc):
    """LSE 800 and 799 overflow exp() unless the max is taken out first."""
    a, b = np.array([[1.0]]), np.array([[0.0]])
    o, lse = orc.merge_splits([a, b], [np.array([800.0]), np.array([799.0])])
    e = math.e
    close(o, [[e / (e + 1.0)]], 1e-14)
    close(lse, [800.0 + math.log1p(1.0 / e)], 1e-15)


# ------------------------------------------------- additive bias ([CSDN] 第一层)

def pin_bias_matches_scalar_brute_force(orc):
    rng = np.random.default_rng(21)
    q, k, v = rng.standard_normal((2, 2, 6, 3)), rng.standard_normal((2, 1, 6, 3)), \
        rng.standard_normal((2, 1, 6, 2))
    bias = 2.0 * rng.standard_normal((2, 2, 6, 6))
    bias[0, 1, 2, 1] = -math.inf  # a bias of −inf removes that key
    for causal, lens in itertools.product([False, True], [None, [4, 0]]):
        o, lse = orc.attention(q, k, v, 0.8, causal, lens, bias=bias)
        ob, lseb = brute_force(q, k, v, 0.8, causal, lens, bias=bias)
        close(o, ob)
        close(lse, lseb)


def pin_bias_matches_torch_sdpa_float_mask(orc):
    """torch's math SDPA adds a float attn_mask to the scaled scores."""
    rng = np.random.default_rng(22)
    B, Hq, Hk, N, d = 2, 4, 2, 19, 8
    q, k, v = rng.standard_normal((B, Hq, N, d)), rng.standard_normal((B, Hk, N, d)), \
        rng.standard_normal((B, Hk, N, d))
    bias = rng.standard_normal((B, Hq, N, N))
    o, _ = orc.attention(q, k, v, 0.4, True, None, bias=bias)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    mask = torch.from_numpy(np.where(j <= i, bias, -np.inf))
    kt = torch.from_numpy(k).repeat_interleave(Hq // Hk, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(Hq // Hk, dim=1)
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), kt, vt, attn_mask=mask, scale=0.4).numpy()
    close(o, ref, 1e-12)


def pin_bias_constant_per_row_shifts_lse_only(orc):
    rng = np.random.default_rng(23)
    q, k, v = rng.standard_normal((1, 2, 9, 4)), rng.standard_normal((1, 2, 9, 4)), \
        rng.standard_normal((1, 2, 9, 4))
    c = rng.standard_normal((1, 2, 9, 1)) * 5.0
    bias = np.broadcast_to(c, (1, 2, 9, 9)).copy()
    o0, l0 = orc.attention(q, k, v, 0.5, True, [7])
    o1, l1 = orc.attention(q, k, v, 0.5, True, [7], bias=bias)
    close(o1, o0, 1e-12)
    close(l1, l0 + c[..., 0], 1e-12)


def pin_bias_minus_inf_equals_key_padding(orc):
    rng = np.random.default_rng(24)
    q, k, v = rng.standard_normal((2, 1, 8, 3)), rng.standard_normal((2, 1, 8, 3)), \
        rng.standard_normal((2, 1, 8, 3))
    lens = [5, 2]
    bias = np.zeros((2, 1, 8, 8))
    for b, L in enumerate(lens):
        bias[b, :, :, L:] = -math.inf
    o0, l0 = orc.attention(q, k, v, 0.9, False, lens)
    o1, l1 = orc.attention(q, k, v, 0.9, False, None, bias=bias)
    close(o1, o0, 1e-12)
    close(l1, l0, 1e-12)


def pin_bias_broadcast_equals_repeated(orc):
    rng = np.random.default_rng(25)
    B, Hq, N = 2, 3, 7
    q, k, v = rng.standard_normal((B, Hq, N, 4)), rng.standard_normal((B, 1, N, 4)), \
        rng.standard_normal((B, 1, N, 4))
    for shape in [(1, 1), (1, Hq), (B, 1)]:
        bias = rng.standard_normal(shape + (N, N))
        full = np.broadcast_to(bias, (B, Hq, N, N)).copy()
        o0, l0 = orc.attention(q, k, v, 0.7, True, None, bias=full)
        o1, l1 = orc.attention(q, k, v, 0.7, True, None, bias=bias)
        close(o1, o0, 1e-12)
        close(l1, l0, 1e-12)
        picks = [(b, h, i) for b in range(B) for h in range(Hq) for i in (0, 3, N - 1)]
        orow, lrow = orc.attention_rows(q, k, v, 0.7, True, None, picks, bias=bias)
        idx = tuple(np.array(picks).T)
        close(orow, o0[idx], 1e-12)
        close(lrow, l0[idx], 1e-12)


# ------------------------------------------------------- backward ([NPU] v2)

def _bwd_problem(rng, B=2, Hq=4, Hk=2, N=9, d=5):
    q, k, v, do = (rng.standard_normal(sh) for sh in
                   [(B, Hq, N, d), (B, Hk, N, d), (B, Hk, N, d), (B, Hq, N, d)])
    return q, k, v, do


def pin_backward_matches_torch_autograd(orc):
    """torch float64 math SDPA differentiated by autograd (no empty rows)."""
    rng = np.random.default_rng(31)
    for causal, G, lens in [(False, 1, None), (True, 2, [9, 4]), (False, 4, [3, 9]), (True, 1, None)]:
        B, Hk, N, d = 2, 2, 9, 5
        q, k, v, do = _bwd_problem(rng, B, Hk * G, Hk, N, d)
        o, lse = orc.attention(q, k, v, 0.6, causal, lens)
        dq, dk, dv = orc.attention_backward(q, k, v, o, lse, do, 0.6, causal, lens)
        tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
        i = torch.arange(N)[:, None]
        j = torch.arange(N)[None, :]
        mask = torch.stack([(j < (N if lens is None else L)) & ((j <= i) if causal else (j >= 0))
                            for L in (lens or [N] * B)])[:, None]
        with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
            out = torch.nn.functional.scaled_dot_product_attention(
                tq, tk.repeat_interleave(G, dim=1), tv.repeat_interleave(G, dim=1),
                attn_mask=mask, scale=0.6)
        (out * torch.from_numpy(do)).sum().backward()
        close(dq, tq.grad.numpy(), 1e-11)
        close(dk, tk.grad.numpy(), 1e-11)
        close(dv, tv.grad.numpy(), 1e-11)


def pin_backward_finite_differences(orc):
    """Central differences of L = Σ dO ⊙ O through the (separately pinned) forward."""
    rng = np.random.default_rng(32)
    q, k, v, do = _bwd_problem(rng, 1, 2, 1, 6, 3)
    lens = [5]
    o, lse = orc.attention(q, k, v, 0.8, True, lens)
    grads = orc.attention_backward(q, k, v, o, lse, do, 0.8, True, lens)
    h = 1e-6
    for which, x in enumerate((q, k, v)):
        for idx in [(0, 0, 0, 0), (0, 0, 3, 2), (0, x.shape[1] - 1, 5, 1), (0, 0, 2, 1)]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = [q, k, v]
            args[which] = xp
            lp = np.sum(do * orc.attention(*args, 0.8, True, lens)[0])
            args[which] = xm
            lm = np.sum(do * orc.attention(*args, 0.8, True, lens)[0])
            assert abs((lp - lm) / (2 * h) - grads[which][idx]) < 1e-7


def pin_backward_closed_form_at_zero_scale(orc):
    """scale = 0: P is uniform over the allowed keys, so dV_j = Σ_i dO_i / L_i over
    the rows i that allow key j, and dQ = dK = 0."""
    rng = np.random.default_rng(33)
    q, k, v, do = _bwd_problem(rng, 1, 2, 2, 7, 3)
    o, lse = orc.attention(q, k, v, 0.0, True, [5])
    dq, dk, dv = orc.attention_backward(q, k, v, o, lse, do, 0.0, True, [5])
    close(dq, np.zeros_like(dq), 0)
    close(dk, np.zeros_like(dk), 0)
    want = np.zeros_like(dv)
    for h in range(2):
        for i in range(7):
            n_allowed = min(i + 1, 5)
            for j in range(n_allowed):
                want[0, h, j] += do[0, h, i] / n_allowed
    close(dv, want, 1e-13)


def pin_backward_empty_rows_and_gqa_sum(orc):
    """A batch with no valid key passes no gradient; GQA dK, dV equal the sum
    over the group of the gradients taken with K, V repeated per query head."""
    rng = np.random.default_rng(34)
    q, k, v, do = _bwd_problem(rng, 2, 4, 2, 6, 3)
    lens = [0, 4]
    o, lse = orc.attention(q, k, v, 0.9, False, lens)
    dq, dk, dv = orc.attention_backward(q, k, v, o, lse, do, 0.9, False, lens)
    assert not dq[0].any() and not dk[0].any() and not dv[0].any()
    kr, vr = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    o2, lse2 = orc.attention(q, kr, vr, 0.9, False, lens)
    dq2, dk2, dv2 = orc.attention_backward(q, kr, vr, o2, lse2, do, 0.9, False, lens)
    close(dq, dq2, 1e-13)
    close(dk, dk2.reshape(2, 2, 2, 6, 3).sum(axis=2), 1e-13)
    close(dv, dv2.reshape(2, 2, 2, 6, 3).sum(axis=2), 1e-13)


def pin_hand_worked_golden(orc):
    """Problems worked by hand (tests/golden/hand_worked.json) to closed-form values."""
    for c in load_golden():
        o, lse = orc.attention(c["q"], c["k"], c["v"], c["scale"], c["causal"], c["key_pad_lens"])
        close(o, c["o"], 1e-14)
        close(lse, c["lse"], 1e-14)


PINS = [f for name, f in sorted(globals().items()) if name.startswith("pin_")]
