"""fp64 CPU oracle for fused online-softmax attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg
and ``--impl reference``) may import this module.  The library itself never does:
the CUDA path must not route through here.

What it computes, for every batch b, query head h and query row i:

    kvh   = h // G,  G = Hq // Hkv          (consecutive query heads share a KV head:
                                              TurboQuant "Attention API" page,
                                              compute_hybrid_attention_store, the
                                              (T, H_kv, G, D) view of the query)
    V_i   = { j < Sk : not causal  or  j <= i + Sk - Sq }   (bottom-right causal
                                              alignment; the pages only use Sq == Sk,
                                              where every alignment agrees)
    s_j   = scale * sum_d q[b,i,h,d] * k[b,j,kvh,d]
    M     = max_{j in V_i} s_j                (explicit max subtraction)
    Z     = sum_{j in V_i} exp(s_j - M)
    O     = sum_{j in V_i} exp(s_j - M) * v[b,j,kvh,:] / Z
    LSE   = M + log Z                          (natural log; StreamAttention page,
                                              "Kernel Design": lse = running max +
                                              log of the running denominator)
    empty V_i  ->  O = 0, LSE = -inf           (TurboQuant page: no keys gives zeros)

The StreamAttention page's online recurrence ("Kernel Design (Fused Online
Softmax)") is an exact reordering of this normalisation, so the direct definition
is the oracle; :func:`attention_blockwise` restates the recurrence itself (the
TurboQuant page's ``online_softmax_attention`` loop) so a test can pin the two
against each other.  Everything is float64; inputs are widened exactly from
their storage dtype.  No blocking, fusion or reordering beyond what is stated.
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _visible(Sq, Sk, causal, rows=None):
    """Boolean [len(rows), Sk] visibility mask (bottom-right causal alignment)."""
    rows = np.arange(Sq) if rows is None else np.asarray(rows)
    j = np.arange(Sk)
    if not causal:
        return np.ones((rows.size, Sk), dtype=bool)
    return j[None, :] <= (rows[:, None] + (Sk - Sq))


def _softmax_attend(qm, km, vm, scale, vis):
    """Plain softmax attention for one (batch, head): qm [n, D], km/vm [Sk, D],
    vis [n, Sk].  Returns O [n, D] and LSE [n] in float64."""
    s = scale * (qm @ km.T)                      # scores, [n, Sk]
    s = np.where(vis, s, NEG_INF)
    n = qm.shape[0]
    o = np.zeros((n, vm.shape[1]), dtype=np.float64)
    lse = np.full(n, NEG_INF, dtype=np.float64)
    has = vis.any(axis=1)
    if has.any():
        sh = s[has]
        m = sh.max(axis=1)                       # M
        e = np.exp(sh - m[:, None])              # exp(s_j - M), 0 for masked keys
        z = e.sum(axis=1)                        # Z
        o[has] = (e @ vm) / z[:, None]
        lse[has] = m + np.log(z)
    return o, lse


def attention(q, k, v, scale, causal=False):
    """Full oracle.  q [B,Sq,Hq,D], k/v [B,Sk,Hkv,D] -> (O [B,Sq,Hq,D], LSE [B,Hq,Sq])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if Hkv == 0 or Hq % Hkv:
        raise ValueError("Hq must be a positive multiple of Hkv")
    G = Hq // Hkv
    O = np.zeros((B, Sq, Hq, D), dtype=np.float64)
    LSE = np.full((B, Hq, Sq), NEG_INF, dtype=np.float64)
    if Sq == 0 or Sk == 0:
        return O, LSE
    vis = _visible(Sq, Sk, causal)
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            O[b, :, h, :], LSE[b, h, :] = _softmax_attend(
                q[b, :, h, :], k[b, :, kvh, :], v[b, :, kvh, :], scale, vis)
    return O, LSE


def attention_rows(q, k, v, scale, causal, b, h, rows):
    """Oracle for selected query rows of one (batch, head): returns O [n, D], LSE [n].
    Used where the full Sq x Sk score matrix would not fit (long sequences)."""
    rows = np.asarray(rows, dtype=np.int64)
    Sq, Hq = q.shape[1], q.shape[2]
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    kvh = h // G
    qm = _f64(q[b, rows, h, :])
    if Sk == 0:
        return np.zeros((rows.size, q.shape[3])), np.full(rows.size, NEG_INF)
    vis = _visible(Sq, Sk, causal, rows)
    return _softmax_attend(qm, _f64(k[b, :, kvh, :]), _f64(v[b, :, kvh, :]), scale, vis)


def decode(q, k, v, scale):
    """Single-token decode: q [B,Hq,D], k/v [B,Sk,Hkv,D]; every key is visible.
    Returns O [B,Hq,D] and LSE [B,Hq]."""
    O, LSE = attention(_f64(q)[:, None], k, v, scale, causal=False)
    return O[:, 0], LSE[:, :, 0]


def decode_paged(q, k_cache, v_cache, block_table, seqlens, scale):
    """Single-token decode over a paged K/V cache (the Stem / AngelSlim page, section 2:
    the serving backend's "paged" path; the flash-attn-volta page lists variable-length
    sequences among what it lacks).  q [B,Hq,D]; k_cache/v_cache [num_pages, page_size,
    Hkv, D]; block_table [B, max_blocks]; seqlens [B].  Sequence b's keys are tokens
    0 .. seqlens[b]-1, token t stored in page block_table[b, t // page_size] at row
    t % page_size; the result is :func:`decode` of q[b] over exactly those keys (a length
    of 0 gives O = 0, LSE = -inf).  Lengths are clamped to [0, page_size * max_blocks].
    Returns O [B,Hq,D] and LSE [B,Hq]."""
    q = _f64(q)
    B, Hq, D = q.shape
    page_size = k_cache.shape[1]
    bt = np.asarray(block_table)
    O = np.zeros((B, Hq, D))
    LSE = np.full((B, Hq), NEG_INF)
    for b in range(B):
        n = int(min(max(int(seqlens[b]), 0), page_size * bt.shape[1]))
        if n == 0:
            continue
        t = np.arange(n)
        pages = bt[b, t // page_size]
        kb = _f64(k_cache)[pages, t % page_size]          # [n, Hkv, D] in token order
        vb = _f64(v_cache)[pages, t % page_size]
        o, lse = decode(q[b:b + 1], kb[None], vb[None], scale)
        O[b], LSE[b] = o[0], lse[0]
    return O, LSE


def attention_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale, causal=False):
    """Attention over sequences of different lengths packed back to back (the Stem /
    AngelSlim page, section 2: the serving backend's "varlen" path; the flash-attn-volta
    page lists variable-length sequences among what it lacks).  q [total_q, Hq, D],
    k/v [total_k, Hkv, D]; sequence b owns query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
    and key rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1, and is :func:`attention` of those
    rows alone (batch of one; causal alignment bottom-right within the sequence).
    Returns O [total_q, Hq, D] and LSE [Hq, total_q]; rows outside every sequence stay
    O = 0, LSE = -inf."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq = [int(x) for x in np.asarray(cu_seqlens_q)]
    ck = [int(x) for x in np.asarray(cu_seqlens_k)]
    if len(cq) != len(ck):
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length")
    total_q, Hq, D = q.shape
    O = np.zeros((total_q, Hq, D))
    LSE = np.full((Hq, total_q), NEG_INF)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 <= q0:
            continue
        o, lse = attention(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], scale, causal)
        O[q0:q1], LSE[:, q0:q1] = o[0], lse[0]
    return O, LSE


def attention_block_sparse(q, k, v, block_mask, scale, causal=False, block=128):
    """Block-sparse attention (the Stem / AngelSlim page, section 2.3: attention over
    the key blocks the top-k mask keeps, block_size 128; initial "sink" blocks and the
    sliding-window blocks are among them).  q [B,Sq,Hq,D], k/v [B,Sk,Hkv,D];
    block_mask [B, Hq, ceil(Sq/block), ceil(Sk/block)], nonzero = keep.  Key j is visible
    to query row i of head h iff the dense rule allows it (bottom-right causal alignment
    when causal) AND block_mask[b, h, i // block, j // block] is nonzero; the rest is
    :func:`attention`'s definition (no visible key: O = 0, LSE = -inf).
    Returns O [B,Sq,Hq,D], LSE [B,Hq,Sq]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if Hkv == 0 or Hq % Hkv:
        raise ValueError("Hq must be a positive multiple of Hkv")
    bm = np.asarray(block_mask) != 0
    nq, nk = -(-Sq // block), -(-Sk // block)
    if bm.shape != (B, Hq, nq, nk):
        raise ValueError(f"block_mask must be [{B}, {Hq}, {nq}, {nk}], got {bm.shape}")
    G = Hq // Hkv
    O = np.zeros((B, Sq, Hq, D))
    LSE = np.full((B, Hq, Sq), NEG_INF)
    if Sq == 0 or Sk == 0:
        return O, LSE
    base = _visible(Sq, Sk, causal)
    rows, cols = np.arange(Sq) // block, np.arange(Sk) // block
    for b in range(B):
        for h in range(Hq):
            vis = base & bm[b, h][rows[:, None], cols[None, :]]
            kvh = h // G
            O[b, :, h, :], LSE[b, h, :] = _softmax_attend(
                q[b, :, h, :], k[b, :, kvh, :], v[b, :, kvh, :], scale, vis)
    return O, LSE


def attention_block_sparse_rows(q, k, v, block_mask, scale, causal, b, h, rows, block=128):
    """:func:`attention_block_sparse` for selected query rows of one (batch, head):
    O [n, D], LSE [n].  For sizes whose full score matrix would not fit."""
    rows = np.asarray(rows, dtype=np.int64)
    Sq, Hq = q.shape[1], q.shape[2]
    Sk, Hkv = k.shape[1], k.shape[2]
    kvh = h // (Hq // Hkv)
    if Sk == 0:
        return np.zeros((rows.size, q.shape[3])), np.full(rows.size, NEG_INF)
    bm = np.asarray(block_mask[b, h]) != 0
    vis = _visible(Sq, Sk, causal, rows) & bm[(rows // block)[:, None], (np.arange(Sk) // block)[None, :]]
    return _softmax_attend(_f64(q[b, rows, h, :]), _f64(k[b, :, kvh, :]), _f64(v[b, :, kvh, :]), scale, vis)


def block_sparse_pairs(Sq, Sk, block_mask, causal, block=128):
    """Number of visible (query row, key) pairs under a block mask [.., nq, nk] summed
    over its leading dimensions: the work a block-sparse forward does (4*D FLOP per
    pair).  Counted per kept block from the dense visibility rule."""
    bm = np.asarray(block_mask) != 0
    nq, nk = bm.shape[-2], bm.shape[-1]
    per_block = np.zeros((nq, nk), dtype=np.int64)
    for qi in range(nq):
        r0, r1 = qi * block, min(Sq, (qi + 1) * block)
        for ki in range(nk):
            c0, c1 = ki * block, min(Sk, (ki + 1) * block)
            if not causal:
                per_block[qi, ki] = (r1 - r0) * (c1 - c0)
            else:
                # row i sees keys j <= i + Sk - Sq: clip that bound into the block's columns
                hi = np.clip(np.arange(r0, r1) + Sk - Sq + 1, c0, c1)
                per_block[qi, ki] = int((hi - c0).sum())
    return int((bm.reshape(-1, nq, nk) * per_block[None]).sum())


def attention_backward(q, k, v, do, scale, causal=False):
    """Gradients of the forward's output O with respect to q, k, v for an upstream
    gradient dO (the StreamAttention page, "Backward": recompute the probabilities from the
    saved LSE and stream dQ/dK/dV; the flash-attn-volta page's backward follows the same
    algorithm).  With P = softmax over the visible keys (the forward's rule) and O = P V:
        dV    = P^T dO                       (summed over the query heads of a KV head)
        dP    = dO V^T
        Delta = rowsum(dO * O)  (= rowsum(P * dP))
        dS    = P * (dP - Delta)             (zero at invisible keys)
        dQ    = scale * dS K,   dK = scale * dS^T Q   (dK summed like dV)
    q [B,Sq,Hq,D], k/v [B,Sk,Hkv,D], do [B,Sq,Hq,D].  Returns dQ, dK, dV in float64 with the
    shapes of q, k, v.  Rows without a visible key have P = 0 and contribute nothing."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if Hkv == 0 or Hq % Hkv:
        raise ValueError("Hq must be a positive multiple of Hkv")
    G = Hq // Hkv
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    if Sq == 0 or Sk == 0:
        return dq, dk, dv
    vis = _visible(Sq, Sk, causal)
    has = vis.any(axis=1)
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            qm, km, vm, dom = q[b, :, h, :], k[b, :, kvh, :], v[b, :, kvh, :], do[b, :, h, :]
            s = np.where(vis, scale * (qm @ km.T), NEG_INF)
            p = np.zeros_like(s)
            m = s[has].max(axis=1)
            e = np.exp(s[has] - m[:, None])
            p[has] = e / e.sum(axis=1, keepdims=True)
            o = p @ vm
            dv[b, :, kvh, :] += p.T @ dom
            dp = dom @ vm.T
            delta = (dom * o).sum(axis=1)
            ds = p * (dp - delta[:, None])
            dq[b, :, h, :] = scale * (ds @ km)
            dk[b, :, kvh, :] += scale * (ds.T @ qm)
    return dq, dk, dv


def _probabilities(qm, km, scale, vis):
    """Softmax weights P [n, Sk] of query rows qm [n, D] over keys km [Sk, D] (visible
    where vis [n, Sk]); rows without a visible key get P = 0."""
    s = np.where(vis, scale * (qm @ km.T), NEG_INF)
    p = np.zeros_like(s)
    has = vis.any(axis=1)
    if has.any():
        m = s[has].max(axis=1)
        e = np.exp(s[has] - m[:, None])
        p[has] = e / e.sum(axis=1, keepdims=True)
    return p


def attention_backward_rows(q, k, v, do, scale, causal, b, h, rows):
    """dQ of selected query rows of one (batch, query head), for long sequences where
    :func:`attention_backward`'s full score matrices would not fit.  A row's gradient
    needs only its own softmax row (the StreamAttention page, "Backward": probabilities
    recomputed from the scores): P_i over the visible keys, O_i = P_i V, dP_i = dO_i V^T,
    Delta_i = dO_i . O_i, dS_i = P_i * (dP_i - Delta_i), dQ_i = scale * dS_i K.
    Shapes as :func:`attention_backward`; returns dQ [len(rows), D] in float64."""
    rows = np.asarray(rows, dtype=np.int64)
    Sq, Hq = q.shape[1], q.shape[2]
    Sk, Hkv = k.shape[1], k.shape[2]
    kvh = h // (Hq // Hkv)
    qm, dom = _f64(q[b, rows, h, :]), _f64(do[b, rows, h, :])
    if Sk == 0:
        return np.zeros_like(qm)
    km, vm = _f64(k[b, :, kvh, :]), _f64(v[b, :, kvh, :])
    p = _probabilities(qm, km, scale, _visible(Sq, Sk, causal, rows))
    dp = dom @ vm.T
    delta = (dom * (p @ vm)).sum(axis=1)
    ds = p * (dp - delta[:, None])
    return scale * (ds @ km)


def attention_backward_keys(q, k, v, do, scale, causal, b, kvh, keys):
    """dK and dV of selected keys of one (batch, KV head): the sums over the G query heads
    of the group and over every query row that sees the key (dV_j = sum_i P_ij dO_i,
    dK_j = scale * sum_i dS_ij Q_i, with P, dS of :func:`attention_backward_rows`).  Only
    the rows that see some selected key are formed (causal: rows i >= min(keys) - (Sk - Sq)),
    so keys near the end of a long causal sequence stay cheap.  Returns dK, dV
    [len(keys), D] in float64."""
    keys = np.asarray(keys, dtype=np.int64)
    Sq, Hq, D = q.shape[1], q.shape[2], q.shape[3]
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    dk = np.zeros((keys.size, D))
    dv = np.zeros((keys.size, D))
    if Sq == 0 or keys.size == 0:
        return dk, dv
    first = max(0, int(keys.min()) - (Sk - Sq)) if causal else 0
    rows = np.arange(first, Sq)
    vis = _visible(Sq, Sk, causal, rows)
    km, vm = _f64(k[b, :, kvh, :]), _f64(v[b, :, kvh, :])
    for h in range(kvh * G, (kvh + 1) * G):
        qm, dom = _f64(q[b, rows, h, :]), _f64(do[b, rows, h, :])
        p = _probabilities(qm, km, scale, vis)
        dp = dom @ vm.T
        delta = (dom * (p @ vm)).sum(axis=1)
        ds = p * (dp - delta[:, None])
        dv += p[:, keys].T @ dom
        dk += scale * (ds[:, keys].T @ qm)
    return dk, dv


def decode_e4m3(codes):
    """Values of 8-bit e4m3 codes (sign bit, 4-bit exponent with bias 7, 3-bit mantissa;
    exponent 0 = subnormal m * 2^-9; 0x7f / 0xff = NaN; no infinities; largest 448) as
    float64 -- the FP8 format the Stem page's fp8 prefill path and the StreamAttention
    page's FP8 roadmap item name, written out from its definition."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def attention_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale, causal=False):
    """Attention on FP8 inputs: :func:`attention` of the dequantised tensors
    decode_e4m3(q8) * q_descale, decode_e4m3(k8) * k_descale, decode_e4m3(v8) * v_descale
    (per-tensor descale factors).  Shapes as :func:`attention`."""
    return attention(decode_e4m3(q8) * q_descale, decode_e4m3(k8) * k_descale, decode_e4m3(v8) * v_descale,
                     scale, causal)


def attention_paged_prefill(q, k_cache, v_cache, cu_seqlens_q, block_table, seqlens_k, scale, causal=False):
    """Packed queries against a paged K/V cache (chunked prefill; the Stem / AngelSlim page's
    serving backend, "varlen" and "paged" paths).  q [total_q, Hq, D]; k_cache/v_cache
    [num_pages, page_size, Hkv, D]; sequence b owns query rows cu_seqlens_q[b] ..
    cu_seqlens_q[b+1]-1 and keys 0 .. seqlens_k[b]-1, key t in page block_table[b, t //
    page_size] at row t % page_size (lengths clamped to the table).  Each sequence is
    :func:`attention` of its rows and its gathered keys (causal bottom-right within it).
    Returns O [total_q, Hq, D], LSE [Hq, total_q]; rows outside every sequence: 0 / -inf."""
    q = _f64(q)
    cq = [int(x) for x in np.asarray(cu_seqlens_q)]
    bt = np.asarray(block_table)
    page_size = k_cache.shape[1]
    total_q, Hq, D = q.shape
    O = np.zeros((total_q, Hq, D))
    LSE = np.full((Hq, total_q), NEG_INF)
    for b in range(len(cq) - 1):
        q0, q1 = cq[b], cq[b + 1]
        if q1 <= q0:
            continue
        n = int(min(max(int(seqlens_k[b]), 0), page_size * bt.shape[1]))
        t = np.arange(n)
        kb = _f64(k_cache)[bt[b, t // page_size], t % page_size]    # [n, Hkv, D] in key order
        vb = _f64(v_cache)[bt[b, t // page_size], t % page_size]
        o, lse = attention(q[None, q0:q1], kb[None], vb[None], scale, causal)
        O[q0:q1], LSE[:, q0:q1] = o[0], lse[0]
    return O, LSE


def attention_blockwise(q, k, v, scale, causal=False, block=64):
    """The online-softmax recurrence, restated in float64 (TurboQuant page,
    ``online_softmax_attention``; StreamAttention page, "Kernel Design"): walk the
    keys in blocks, keep a running max m, running denominator l and accumulator acc,
    rescale both by exp(m_old - m_new) when the max grows, finish with acc / l.
    A fully masked block leaves the state unchanged (the flash-attn-volta page's
    fully-masked-row guard: exponentiate against 0 while the max is still -inf)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    O = np.zeros((B, Sq, Hq, D))
    LSE = np.full((B, Hq, Sq), NEG_INF)
    vis = _visible(Sq, Sk, causal)
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            qm = q[b, :, h, :]
            m = np.full(Sq, NEG_INF)
            l = np.zeros(Sq)
            acc = np.zeros((Sq, D))
            for start in range(0, Sk, block):
                end = min(start + block, Sk)
                s = scale * (qm @ k[b, start:end, kvh, :].T)
                s = np.where(vis[:, start:end], s, NEG_INF)
                m_new = np.maximum(m, s.max(axis=1))
                ref = np.where(np.isneginf(m_new), 0.0, m_new)   # the guard
                alpha = np.exp(m - ref)
                p = np.exp(s - ref[:, None])
                l = l * alpha + p.sum(axis=1)
                acc = acc * alpha[:, None] + p @ v[b, start:end, kvh, :]
                m = m_new
            ok = l > 0
            O[b, ok, h, :] = acc[ok] / l[ok, None]
            LSE[b, h, ok] = m[ok] + np.log(l[ok])
    return O, LSE


def combine_lse(outs, lses):
    """LSE-weighted merge of partial attention results over disjoint key sets
    (StreamAttention page, "Distributed and Long-Context Variants": log-sum-exp
    weighted combining; its "Engine Direction" section: partial online-softmax
    states merged in a second kernel).  outs[s] [..., D] normalised partial outputs,
    lses[s] [...] their natural-log LSEs.  Parts with LSE = -inf carry no weight."""
    lses = np.stack([_f64(x) for x in lses])          # [S, ...]
    outs = np.stack([_f64(x) for x in outs])          # [S, ..., D]
    mx = lses.max(axis=0)
    ref = np.where(np.isneginf(mx), 0.0, mx)
    w = np.exp(lses - ref)                            # [S, ...]
    den = w.sum(axis=0)
    lse = np.where(den > 0, ref + np.log(np.where(den > 0, den, 1.0)), NEG_INF)
    o = np.where((den > 0)[..., None],
                 (w[..., None] * outs).sum(axis=0) / np.where(den > 0, den, 1.0)[..., None], 0.0)
    return o, lse
