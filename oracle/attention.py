"""Float64 CPU oracle for the exact attention forward pass.

TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the CPU-baseline leg of
the benchmark may import this module; the product path (the C-ABI library and
its Python binding) never does, and this module imports nothing from it.

What it computes, and where the pages say so (page title, then section):

* [FA-VI] "FlashAttention (VI)", section "Vấn đề của cơ chế attention tiêu
  chuẩn": Attention(Q, K, V) = softmax(Q Kᵀ / sqrt(d_k)) V, with the full N×N
  score matrix S formed first.
* [MCU] "MCU 上 Transformer 模型的 Flash Attention 实现在 256KB SRAM 约束下的分块
  计算与内存建模方案", §二: the plain softmax takes two passes (row max, then
  the sum of exp(x − max)); the same section gives the online recurrence
  (running max m, running denominator l, rescaled O) and states that the final
  O / l equals full softmax attention exactly. §三 ends with the division by l
  and a guard for rows whose l is zero.
* [NPU] "FlashAttention 在昇腾 NPU 上是怎么省显存的？我花了两天把它搞明白了",
  "坑一" (generation models use a causal mask, BERT-style models do not) and
  "坑四" (GQA/MQA: K and V carry fewer heads than Q).
* [CSDN] aicoding.csdn.net page on ops-transformer FlashAttention, "第一层，
  算子融合": the mask is applied inside the fused kernel.
* [CSDN] "第一层，算子融合" also lists Bias among the operations fused into
  the kernel (beside Dropout and Mask), without giving its shape. Read here as
  an additive term on the scaled scores, S = scale·Q Kᵀ + bias, with bias of
  shape [Bb, Hb, N, N] broadcast over batch (Bb = 1) and heads (Hb = 1); the
  mask applies after it.
* [NPU] (section before "实际跑一下"): standard attention keeps S and P for the
  backward pass; the v2 FlashAttention reworks the gradient computation to
  use less memory. No formulas are given. Read here as the gradient of the
  forward definition above (dQ, dK, dV for a given dO), with P rebuilt from
  Q, K and the forward's LSE instead of stored: P = exp(S − LSE).
* [GQA] "深度探索Flash-Attention中GQA性能调优技术解析", section
  "num_splits参数的场景化配置": the attention work of one problem may be cut
  into num_splits parts. Read here as a split of the key range, each part's
  result merged by its log-sum-exp (the section gives no formula; the merge is
  the [MCU] §二 recurrence with a whole key range as one tile).

Readings taken where the pages are silent or garbled: the mask is additive
−inf after scaling; causal allows key j when
j <= i; key padding removes keys j >= L_b and still computes every query row;
LSE_i = ln Σ_j exp(scale·q_i·k_j) over allowed j; query head hq reads K/V head
hq // (Hq / Hk); a row with no allowed key has O = 0 and LSE = −inf.

All arithmetic is float64. Inputs are the already-rounded fp16/bf16 values,
converted exactly to float64 by the caller (every fp16/bf16 value is a float64).
"""

import numpy as np

__all__ = [
    "allowed_keys",
    "scores",
    "two_pass_softmax",
    "attention",
    "attention_rows",
    "online_attention_flowchart",
    "online_attention_equations",
    "attention_key_range",
    "merge_splits",
    "split_kv_attention",
    "attention_backward",
]


def allowed_keys(rows, n_keys, causal, key_len):
    """Boolean matrix allowed[r, j] for query rows `rows` and keys 0..n_keys-1.

    A key is allowed when it is a real (unpadded) key, j < key_len, and, with
    the causal mask of [NPU] "坑一", when it is not in the future: j <= i.
    """
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(n_keys, dtype=np.int64)[None, :]
    ok = (j < key_len) & (i >= 0)
    if causal:
        ok = ok & (j <= i)
    return ok


def scores(q_rows, k, scale, ok, bias_rows=None):
    """S = scale · Q Kᵀ (+ bias) for the given query rows, −inf where not allowed.

    [FA-VI]: the scores of standard attention; [CSDN]: the mask (and an
    additive bias, not scaled) are part of the same fused computation, the
    mask taken here as an additive −inf.
    """
    s = scale * (q_rows @ k.T)
    if bias_rows is not None:
        s = s + bias_rows
    return np.where(ok, s, -np.inf)


def _bias_slice(bias, b, hq):
    """The [N, N] bias plane of (b, hq): bias is [Bb, Hb, N, N] with Bb in {1, B}
    and Hb in {1, Hq} (size-1 dimensions broadcast), or None."""
    if bias is None:
        return None
    return bias[b if bias.shape[0] > 1 else 0, hq if bias.shape[1] > 1 else 0]


def two_pass_softmax(s):
    """Row softmax of S in the two passes of [MCU] §二.

    Pass 1 takes the row max m; pass 2 takes p = exp(s − m) and l = Σ p.
    Returns (p, m, l). A row with no finite entry has p = 0, m = −inf, l = 0.
    """
    m = s.max(axis=1)
    has = np.isfinite(m)
    m_safe = np.where(has, m, 0.0)
    p = np.where(np.isfinite(s), np.exp(s - m_safe[:, None]), 0.0)
    l = p.sum(axis=1)
    return p, m, l


def _finish(p, m, l, v):
    """O = (P V) / l and LSE = m + ln l, per [MCU] §三's final division by l.

    Rows with l = 0 (no allowed key) get O = 0 and LSE = −inf.
    """
    has = l > 0.0
    o = np.zeros((p.shape[0], v.shape[1]), dtype=np.float64)
    o[has] = (p[has] @ v) / l[has][:, None]
    lse = np.full(p.shape[0], -np.inf, dtype=np.float64)
    lse[has] = m[has] + np.log(l[has])
    return o, lse


def _as_f64(x):
    return np.asarray(x, dtype=np.float64)


def _key_len(key_pad_lens, b, n):
    if key_pad_lens is None:
        return n
    return int(min(max(int(key_pad_lens[b]), 0), n))


def attention(q, k, v, scale, causal=False, key_pad_lens=None, row_block=1024, bias=None):
    """Exact attention forward: returns (O [B,Hq,N,d], LSE [B,Hq,N]) in float64.

    q: [B, Hq, N, d]; k, v: [B, Hk, N, d]; key_pad_lens: None or [B] integers;
    bias: None or [Bb, Hb, N, N] (see _bias_slice).
    Each row block holds full rows of S (all N keys), so the result is the
    plain definition of [FA-VI] with the two-pass softmax of [MCU] §二; the
    blocking over rows only bounds memory, as rows are independent.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    bias = None if bias is None else _as_f64(bias)
    B, Hq, N, d = q.shape
    Hk = k.shape[1]
    if Hq % Hk != 0:
        raise ValueError("Hq must be a multiple of Hk")
    group = Hq // Hk
    o = np.zeros((B, Hq, N, v.shape[3]), dtype=np.float64)
    lse = np.full((B, Hq, N), -np.inf, dtype=np.float64)
    for b in range(B):
        key_len = _key_len(key_pad_lens, b, N)
        for hq in range(Hq):
            hk = hq // group  # [NPU] "坑四": a K/V head serves Hq/Hk query heads
            plane = _bias_slice(bias, b, hq)
            for r0 in range(0, N, row_block):
                rows = np.arange(r0, min(r0 + row_block, N))
                ok = allowed_keys(rows, N, causal, key_len)
                s = scores(q[b, hq, rows], k[b, hk], scale, ok,
                           None if plane is None else plane[rows])
                p, m, l = two_pass_softmax(s)
                o[b, hq, rows], lse[b, hq, rows] = _finish(p, m, l, v[b, hk])
    return o, lse


def attention_rows(q, k, v, scale, causal, key_pad_lens, picks, bias=None):
    """The same definition for selected rows only.

    picks: iterable of (b, hq, i). Returns (O [len(picks), d], LSE [len(picks)]).
    Used to check full-size problems on sampled outputs.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    _, Hq, N, _ = q.shape
    group = Hq // k.shape[1]
    picks = list(picks)
    o = np.zeros((len(picks), v.shape[3]), dtype=np.float64)
    lse = np.zeros(len(picks), dtype=np.float64)
    for n, (b, hq, i) in enumerate(picks):
        hk = hq // group
        ok = allowed_keys([i], N, causal, _key_len(key_pad_lens, b, N))
        plane = _bias_slice(bias, b, hq)
        s = scores(q[b, hq, [i]], k[b, hk], scale, ok,
                   None if plane is None else _as_f64(plane[[i]]))
        p, m, l = two_pass_softmax(s)
        o1, lse1 = _finish(p, m, l, v[b, hk])
        o[n], lse[n] = o1[0], lse1[0]
    return o, lse


def _online(q, k, v, scale, causal, key_pad_lens, tile_r, tile_c, update):
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, N, _ = q.shape
    group = Hq // k.shape[1]
    dv = v.shape[3]
    o = np.zeros((B, Hq, N, dv), dtype=np.float64)
    lse = np.full((B, Hq, N), -np.inf, dtype=np.float64)
    for b in range(B):
        key_len = _key_len(key_pad_lens, b, N)
        for hq in range(Hq):
            hk = hq // group
            for r0 in range(0, N, tile_r):
                rows = np.arange(r0, min(r0 + tile_r, N))
                m = np.full(len(rows), -np.inf)
                l = np.zeros(len(rows))
                acc = np.zeros((len(rows), dv))
                for c0 in range(0, N, tile_c):
                    cols = np.arange(c0, min(c0 + tile_c, N))
                    ok = allowed_keys(rows, N, causal, key_len)[:, cols]
                    s = scores(q[b, hq, rows], k[b, hk, cols], scale, ok)
                    m, l, acc = update(m, l, acc, s, v[b, hk, cols])
                has = l > 0.0
                o[b, hq, rows[has]] = acc[has] / l[has][:, None]
                lse[b, hq, rows[has]] = m[has] + np.log(l[has])
    return o, lse


def _exp_diff(a, b):
    """exp(a − b) with the convention exp(−inf − (−inf)) = 0 (nothing seen yet)."""
    a, b = np.broadcast_arrays(a, b)
    both_inf = np.isneginf(a) & np.isneginf(b)
    diff = np.zeros(a.shape)
    np.subtract(a, b, out=diff, where=~both_inf)
    return np.where(both_inf, 0.0, np.exp(diff))


def _update_flowchart(m_old, l_old, o_old, s, v_tile):
    """One K/V tile of [MCU] §二's flowchart.

    m_new = max(m_old, rowmax S); P = exp(S − m_new);
    l_new = exp(m_old − m_new)·l_old + rowsum P;
    O_new = diag(exp(m_old − m_new))·O_old + P V.
    """
    m_new = np.maximum(m_old, s.max(axis=1))
    p = _exp_diff(s, m_new[:, None])
    alpha = _exp_diff(m_old, m_new)
    l_new = alpha * l_old + p.sum(axis=1)
    o_new = alpha[:, None] * o_old + p @ v_tile
    return m_new, l_new, o_new


def _update_equations(m_old, l_old, o_old, s, v_tile):
    """One K/V tile of [MCU] §二's displayed equations (local-max form).

    With m̃ = rowmax S and P̃ = exp(S − m̃):
    m_new = max(m_old, m̃);
    l_new = exp(m_old − m_new)·l_old + exp(m̃ − m_new)·rowsum P̃;
    O_new = exp(m_old − m_new)·O_old + exp(m̃ − m_new)·P̃ V.
    (The page's LaTeX lost its '=' and '+' signs; this is the reading that
    its flowchart and its exactness claim support.)
    """
    m_loc = s.max(axis=1)
    p_loc = _exp_diff(s, m_loc[:, None])
    m_new = np.maximum(m_old, m_loc)
    a_old = _exp_diff(m_old, m_new)
    a_loc = _exp_diff(m_loc, m_new)
    l_new = a_old * l_old + a_loc * p_loc.sum(axis=1)
    o_new = a_old[:, None] * o_old + a_loc[:, None] * (p_loc @ v_tile)
    return m_new, l_new, o_new


def online_attention_flowchart(q, k, v, scale, causal=False, key_pad_lens=None,
                               tile_r=32, tile_c=32):
    """Tiled attention with the online recurrence of [MCU] §二 (flowchart form).

    Each Q tile of tile_r rows keeps its own m, l and O while it visits every
    K/V tile of tile_c keys in order. Used only to check the recurrence
    against the two-pass definition.
    """
    return _online(q, k, v, scale, causal, key_pad_lens, tile_r, tile_c,
                   _update_flowchart)


def online_attention_equations(q, k, v, scale, causal=False, key_pad_lens=None,
                               tile_r=32, tile_c=32):
    """Tiled attention with the online recurrence of [MCU] §二 (equation form)."""
    return _online(q, k, v, scale, causal, key_pad_lens, tile_r, tile_c,
                   _update_equations)


def attention_key_range(q, k, v, scale, causal, key_pad_lens, key_lo, key_hi):
    """Attention with only keys key_lo <= j < key_hi allowed (one part of [GQA]'s split).

    The same definition as `attention`, with the key range as one more mask
    term. Returns (O_s, LSE_s): O_s is normalised by this range's own
    denominator; a row with no allowed key in the range has O_s = 0 and
    LSE_s = −inf.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, N, _ = q.shape
    group = Hq // k.shape[1]
    o = np.zeros((B, Hq, N, v.shape[3]), dtype=np.float64)
    lse = np.full((B, Hq, N), -np.inf, dtype=np.float64)
    j = np.arange(N)[None, :]
    in_range = (j >= key_lo) & (j < key_hi)
    for b in range(B):
        key_len = _key_len(key_pad_lens, b, N)
        for hq in range(Hq):
            hk = hq // group
            rows = np.arange(N)
            ok = allowed_keys(rows, N, causal, key_len) & in_range
            s = scores(q[b, hq], k[b, hk], scale, ok)
            p, m, l = two_pass_softmax(s)
            o[b, hq], lse[b, hq] = _finish(p, m, l, v[b, hk])
    return o, lse


def merge_splits(o_parts, lse_parts):
    """Result over the union of disjoint key ranges from each range's (O_s, LSE_s).

    With m = max_s LSE_s and w_s = exp(LSE_s − m) (0 for LSE_s = −inf):
    O = Σ_s w_s O_s / Σ_s w_s and LSE = m + ln Σ_s w_s. Since LSE_s = m_s +
    ln l_s, w_s is l_s·exp(m_s − m): the [MCU] §二 update of m, l and the
    unnormalised O with one range as the tile. Rows with no allowed key in
    any range get O = 0 and LSE = −inf.
    """
    o_parts = [_as_f64(x) for x in o_parts]
    lse_parts = [_as_f64(x) for x in lse_parts]
    m = np.max(np.stack(lse_parts), axis=0)
    has = np.isfinite(m)
    m_safe = np.where(has, m, 0.0)
    num = np.zeros(o_parts[0].shape)
    den = np.zeros(m.shape)
    for o_s, lse_s in zip(o_parts, lse_parts):
        w = np.where(np.isfinite(lse_s), np.exp(np.where(np.isfinite(lse_s), lse_s, 0.0) - m_safe), 0.0)
        num += w[..., None] * o_s
        den += w
    o = np.zeros(num.shape)
    o[has] = num[has] / den[has][..., None]
    lse = np.full(m.shape, -np.inf)
    lse[has] = m[has] + np.log(den[has])
    return o, lse


def split_kv_attention(q, k, v, scale, causal, key_pad_lens, bounds):
    """[GQA]'s split: keys cut at `bounds` (0 = c_0 < c_1 < ... = N), merged by LSE."""
    parts = [attention_key_range(q, k, v, scale, causal, key_pad_lens, lo, hi)
             for lo, hi in zip(bounds[:-1], bounds[1:])]
    return merge_splits([p[0] for p in parts], [p[1] for p in parts])


def attention_backward(q, k, v, o, lse, do, scale, causal=False, key_pad_lens=None):
    """Gradients (dQ, dK, dV) of O = softmax(scale·QKᵀ + mask)·V for upstream dO.

    The chain rule through the definition, row by row ([NPU] backward reading):
    P = exp(S − LSE) with S the masked scores and LSE the forward's per-row
    log-sum-exp (so P is the forward's softmax, rebuilt, not stored);
    dV = Pᵀ dO; dP = dO Vᵀ; D_i = Σ_c dO_ic O_ic (= Σ_j P_ij dP_ij);
    dS = P ⊙ (dP − D); dQ = scale · dS K; dK = scale · dSᵀ Q. A K/V head
    shared by G query heads ([NPU] "坑四") receives the sum of their dK, dV.
    Rows with no allowed key (LSE = −inf) have P = 0 and pass no gradient.
    """
    q, k, v, o, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(o), _as_f64(do)
    lse = _as_f64(lse)
    B, Hq, N, d = q.shape
    Hk = k.shape[1]
    group = Hq // Hk
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    rows = np.arange(N)
    for b in range(B):
        key_len = _key_len(key_pad_lens, b, N)
        ok = allowed_keys(rows, N, causal, key_len)
        for hq in range(Hq):
            hk = hq // group
            s = scores(q[b, hq], k[b, hk], scale, ok)
            has = np.isfinite(lse[b, hq])
            p = np.zeros((N, N))
            p[has] = np.exp(s[has] - lse[b, hq][has][:, None])
            dv[b, hk] += p.T @ do[b, hq]
            dp = do[b, hq] @ v[b, hk].T
            dsum = np.sum(do[b, hq] * o[b, hq], axis=1)
            ds = p * (dp - dsum[:, None])
            dq[b, hq] = scale * (ds @ k[b, hk])
            dk[b, hk] += scale * (ds.T @ q[b, hq])
    return dq, dk, dv
