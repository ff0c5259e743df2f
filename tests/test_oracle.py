"""Pins for the fp64 oracle: closed forms, invariants and brute force.

Each test fixes the oracle against something other than itself, chosen so that a
plausible slip (a dropped scale, a wrong sign, a transposed operand, a wrong GQA
index or causal offset, a missing max-subtraction guard) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import (attention, attention_rows, attention_blockwise, attention_varlen, attention_block_sparse,
                    attention_block_sparse_rows, block_sparse_pairs, attention_backward, decode, decode_paged,
                    combine_lse)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-12


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def qkv(B=2, Sq=9, Sk=11, Hq=4, Hkv=2, D=8, seed=0, s=1.0):
    return (rnd((B, Sq, Hq, D), seed, s), rnd((B, Sk, Hkv, D), seed + 1, s),
            rnd((B, Sk, Hkv, D), seed + 2, s))


def visible_count(i, Sq, Sk, causal):
    return Sk if not causal else max(0, min(Sk, i + Sk - Sq + 1))


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    q = np.array(g["q"])[None, :, None, :]
    k = np.array(g["k"])[None, :, None, :]
    v = np.array(g["v"])[None, :, None, :]
    for mode, causal in (("noncausal", False), ("causal", True)):
        O, L = attention(q, k, v, g["scale"], causal)
        np.testing.assert_allclose(O[0, :, 0, :], g[mode]["O"], atol=1e-14)
        np.testing.assert_allclose(L[0, 0], g[mode]["LSE"], atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(7, 7), (5, 9), (9, 5)])
def test_zero_query_gives_mean_of_visible_values(causal, Sq, Sk):
    # all scores equal -> uniform weights over the visible keys
    _, k, v = qkv(Sq=Sq, Sk=Sk)
    q = np.zeros((2, Sq, 4, 8))
    O, L = attention(q, k, v, 0.37, causal)
    for b in range(2):
        for h in range(4):
            for i in range(Sq):
                n = visible_count(i, Sq, Sk, causal)
                if n == 0:
                    assert np.all(O[b, i, h] == 0) and L[b, h, i] == -np.inf
                    continue
                mean = np.mean(v[b, :n, h // 2, :], axis=0)
                np.testing.assert_allclose(O[b, i, h], mean, atol=TOL)
                assert abs(L[b, h, i] - math.log(n)) < TOL


def test_zero_scale_gives_mean_of_values():
    q, k, v = qkv()
    O, L = attention(q, k, v, 0.0, False)
    np.testing.assert_allclose(O, np.broadcast_to(
        np.repeat(v.mean(axis=1), 2, axis=1)[:, None], O.shape), atol=TOL)
    np.testing.assert_allclose(L, math.log(11), atol=TOL)


def test_single_key_returns_its_value():
    q, k, v = qkv(Sk=1)
    scale = 0.41
    O, L = attention(q, k, v, scale, False)
    for b in range(2):
        for h in range(4):
            for i in range(9):
                np.testing.assert_allclose(O[b, i, h], v[b, 0, h // 2], atol=TOL)
                ref = scale * math.fsum(q[b, i, h, d] * k[b, 0, h // 2, d] for d in range(8))
                assert abs(L[b, h, i] - ref) < TOL


def test_one_hot_dominant_score_selects_one_value():
    D, Sk, alpha, beta, scale = 8, 8, 4.0, 5.0, 4.0      # scale*alpha*beta = 80
    k = np.zeros((1, Sk, 1, D))
    for j in range(Sk):
        k[0, j, 0, j] = alpha
    v = rnd((1, Sk, 1, D), 3)
    for jstar in range(Sk):
        q = np.zeros((1, 1, 1, D))
        q[0, 0, 0, jstar] = beta
        O, L = attention(q, k, v, scale, False)
        np.testing.assert_allclose(O[0, 0, 0], v[0, jstar, 0], atol=(Sk - 1) * math.exp(-80) * 10)
        assert abs(L[0, 0, 0] - 80.0) < 1e-12


def test_lse_matches_brute_force_sum_of_exponentials():
    # small scores, so log(sum exp(s)) needs no max-subtraction
    q, k, v = qkv(B=1, Sq=4, Sk=6, Hq=2, Hkv=1, D=5, s=0.5)
    scale = 0.7
    _, L = attention(q, k, v, scale, False)
    for h in range(2):
        for i in range(4):
            tot = math.fsum(math.exp(scale * math.fsum(q[0, i, h, d] * k[0, j, 0, d] for d in range(5)))
                            for j in range(6))
            assert abs(L[0, h, i] - math.log(tot)) < 1e-13


def test_output_matches_brute_force_softmax_weights():
    # V = identity rows: O row i is exactly the softmax probability vector
    Sk = D = 6
    q = rnd((1, 3, 1, D), 11)
    k = rnd((1, Sk, 1, D), 12)
    v = np.eye(Sk)[None, :, None, :]
    scale = 0.9
    O, _ = attention(q, k, v, scale, False)
    for i in range(3):
        e = [math.exp(scale * math.fsum(q[0, i, 0, d] * k[0, j, 0, d] for d in range(D)))
             for j in range(Sk)]
        z = math.fsum(e)
        np.testing.assert_allclose(O[0, i, 0], [x / z for x in e], atol=1e-14)


def test_causal_row_zero_is_first_value():
    q, k, v = qkv(Sq=10, Sk=10)
    scale = 0.3
    O, L = attention(q, k, v, scale, True)
    for b in range(2):
        for h in range(4):
            np.testing.assert_allclose(O[b, 0, h], v[b, 0, h // 2], atol=TOL)
            ref = scale * math.fsum(q[b, 0, h, d] * k[b, 0, h // 2, d] for d in range(8))
            assert abs(L[b, h, 0] - ref) < TOL


@pytest.mark.parametrize("causal", [False, True])
def test_affine_in_values(causal):
    q, k, v = qkv()
    a, c = -1.7, 0.25
    O, L = attention(q, k, v, 0.5, causal)
    O2, L2 = attention(q, k, a * v + c, 0.5, causal)
    np.testing.assert_allclose(O2, a * O + c, atol=1e-12)
    np.testing.assert_array_equal(L, L2)


def test_key_permutation_invariance():
    q, k, v = qkv()
    perm = np.random.default_rng(5).permutation(11)
    O, L = attention(q, k, v, 0.5, False)
    O2, L2 = attention(q, k[:, perm], v[:, perm], 0.5, False)
    np.testing.assert_allclose(O2, O, atol=TOL)
    np.testing.assert_allclose(L2, L, atol=TOL)


@pytest.mark.parametrize("causal", [False, True])
def test_score_shift(causal):
    # k_j += u for every j adds scale*q.u to every score of a row: O unchanged
    q, k, v = qkv()
    u = rnd((2, 1, 2, 8), 9)
    scale = 0.45
    O, L = attention(q, k, v, scale, causal)
    O2, L2 = attention(q, k + u, v, scale, causal)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    shift = scale * np.einsum("bihd,bhd->bhi", q, np.repeat(u[:, 0], 2, axis=1))
    np.testing.assert_allclose(L2, L + shift, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_mha_on_repeated_kv(causal):
    # repeat_kv: KV head j serves query heads j*G .. j*G+G-1
    q, k, v = qkv(Hq=6, Hkv=2)
    O, L = attention(q, k, v, 0.5, causal)
    kk, vv = np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2)
    O2, L2 = attention(q, kk, vv, 0.5, causal)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)
    # and not the interleaved (h % Hkv) mapping
    O3, _ = attention(q, np.tile(k, (1, 1, 3, 1)), np.tile(v, (1, 1, 3, 1)), 0.5, causal)
    assert not np.allclose(O, O3)


def test_split_combine_equals_whole():
    q, k, v = qkv(Sk=13)
    O, L = attention(q, k, v, 0.5, False)
    parts = [(0, 5), (5, 6), (6, 13)]
    outs, lses = zip(*[attention(q, k[:, a:b], v[:, a:b], 0.5, False) for a, b in parts])
    lses = [x.transpose(0, 2, 1) for x in lses]          # [B, Sq, Hq]
    Oc, Lc = combine_lse(outs, lses)
    np.testing.assert_allclose(Oc, O, atol=1e-12)
    np.testing.assert_allclose(Lc, L.transpose(0, 2, 1), atol=1e-12)


def test_combine_ignores_empty_parts():
    o = rnd((3, 4), 1)
    l = rnd((3,), 2)
    Oc, Lc = combine_lse([o, np.zeros((3, 4))], [l, np.full(3, -np.inf)])
    np.testing.assert_allclose(Oc, o, atol=TOL)
    np.testing.assert_allclose(Lc, l, atol=TOL)
    Oc, Lc = combine_lse([o, o], [np.full(3, -np.inf)] * 2)
    assert np.all(Oc == 0) and np.all(Lc == -np.inf)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk,block", [(9, 11, 4), (16, 16, 64), (20, 7, 3), (3, 130, 64)])
def test_blockwise_recurrence_equals_direct(causal, Sq, Sk, block):
    q, k, v = qkv(Sq=Sq, Sk=Sk, s=2.0)
    O, L = attention(q, k, v, 0.6, causal)
    O2, L2 = attention_blockwise(q, k, v, 0.6, causal, block)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(L2, L, atol=1e-12)


def test_causal_leak_rows_ignore_future_keys():
    q, k, v = qkv(Sq=12, Sk=12)
    O, L = attention(q, k, v, 0.5, True)
    for i in range(12):
        k2, v2 = k.copy(), v.copy()
        k2[:, i + 1:] += 100.0
        v2[:, i + 1:] -= 50.0
        O2, L2 = attention(q, k2, v2, 0.5, True)
        np.testing.assert_array_equal(O2[:, :i + 1], O[:, :i + 1])
        np.testing.assert_array_equal(L2[:, :, :i + 1], L[:, :, :i + 1])


def test_empty_and_fully_masked():
    q, k, v = qkv(Sk=0)
    O, L = attention(q, k, v, 0.5, False)
    assert np.all(O == 0) and np.all(L == -np.inf)
    q, k, v = qkv(Sq=9, Sk=4)           # causal, Sq > Sk: rows 0..4 see nothing
    O, L = attention(q, k, v, 0.5, True)
    assert np.all(O[:, :5] == 0) and np.all(L[:, :, :5] == -np.inf)
    assert np.all(np.isfinite(L[:, :, 5:]))
    np.testing.assert_allclose(O[:, 5, :, :], np.repeat(v[:, 0], 2, axis=1), atol=TOL)


def test_decode_is_last_causal_row():
    # bottom-right alignment: a single query sees every key, like the last causal row
    q, k, v = qkv(Sq=6, Sk=6)
    O, L = attention(q, k, v, 0.5, True)
    Od, Ld = decode(q[:, -1], k, v, 0.5)
    np.testing.assert_allclose(Od, O[:, -1], atol=TOL)
    np.testing.assert_allclose(Ld, L[:, :, -1], atol=TOL)
    Oc, Lc = attention(q[:, -1:], k, v, 0.5, True)          # Sq=1 causal == all visible
    np.testing.assert_allclose(Oc[:, 0], Od, atol=TOL)


def test_rows_match_full():
    q, k, v = qkv(Sq=10, Sk=12)
    O, L = attention(q, k, v, 0.5, True)
    rows = [0, 3, 9]
    for b in range(2):
        for h in range(4):
            Or, Lr = attention_rows(q, k, v, 0.5, True, b, h, rows)
            np.testing.assert_allclose(Or, O[b, rows, h], atol=TOL)
            np.testing.assert_allclose(Lr, L[b, h, rows], atol=TOL)


def test_large_scores_stay_finite():
    # max-subtraction: scores ~ 1e3 would overflow exp() without it
    q, k, v = qkv(s=30.0)
    O, L = attention(q, k, v, 1.0, True)
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(L))
    assert np.all(np.abs(O) <= np.abs(v).max() + 1e-9)


# ---- paged decode: a gather by the block table, then the plain decode

def paged_from_dense(k, v, page_size, perm_seed=None):
    """Cut dense [B,Sk,Hkv,D] K/V into pages of page_size rows (Sk a multiple), optionally
    shuffle the pages in the cache, and return (k_cache, v_cache, block_table)."""
    B, Sk, Hkv, D = k.shape
    nb = Sk // page_size
    kc = k.reshape(B * nb, page_size, Hkv, D)
    vc = v.reshape(B * nb, page_size, Hkv, D)
    table = np.arange(B * nb).reshape(B, nb)
    if perm_seed is not None:
        perm = np.random.default_rng(perm_seed).permutation(B * nb)   # page i moves to slot perm[i]
        kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
        kc2[perm], vc2[perm] = kc, vc
        kc, vc, table = kc2, vc2, perm[table]
    return kc, vc, table


def test_paged_decode_identity_layout_is_dense_decode():
    q, k, v = qkv(B=3, Sq=1, Sk=12, Hq=4, Hkv=2)
    kc, vc, table = paged_from_dense(k, v, 4)
    O, L = decode_paged(q[:, 0], kc, vc, table, np.full(3, 12), 0.5)
    Od, Ld = decode(q[:, 0], k, v, 0.5)
    np.testing.assert_allclose(O, Od, atol=TOL)
    np.testing.assert_allclose(L, Ld, atol=TOL)


def test_paged_decode_ignores_where_pages_sit():
    q, k, v = qkv(B=2, Sq=1, Sk=16, Hq=6, Hkv=3, seed=5)
    kc, vc, table = paged_from_dense(k, v, 4, perm_seed=11)
    O, L = decode_paged(q[:, 0], kc, vc, table, np.array([16, 16]), 0.7)
    Od, Ld = decode(q[:, 0], k, v, 0.7)
    np.testing.assert_allclose(O, Od, atol=TOL)
    np.testing.assert_allclose(L, Ld, atol=TOL)


def test_paged_decode_lengths_truncate_and_empty():
    q, k, v = qkv(B=4, Sq=1, Sk=12, Hq=2, Hkv=1, seed=9)
    kc, vc, table = paged_from_dense(k, v, 4, perm_seed=3)
    lens = np.array([12, 5, 0, 1])
    O, L = decode_paged(q[:, 0], kc, vc, table, lens, 0.5)
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(O[b] == 0) and np.all(np.isneginf(L[b]))
            continue
        Od, Ld = decode(q[b:b + 1, 0], k[b:b + 1, :n], v[b:b + 1, :n], 0.5)
        np.testing.assert_allclose(O[b], Od[0], atol=TOL)
        np.testing.assert_allclose(L[b], Ld[0], atol=TOL)
    # one visible key: the output is that key's V row, the LSE its score
    np.testing.assert_allclose(O[3], v[3, 0, [0, 0]], atol=TOL)
    np.testing.assert_allclose(L[3], 0.5 * (q[3, 0] @ k[3, 0, 0]), atol=TOL)
    # lengths beyond the table are clamped to it
    O2, L2 = decode_paged(q[:, 0], kc, vc, table, np.array([99, 5, -3, 1]), 0.5)
    np.testing.assert_allclose(O2[0], O[0], atol=TOL)
    assert np.all(O2[2] == 0) and np.all(np.isneginf(L2[2]))


# ---- variable-length sequences packed back to back

def packed(lens_q, lens_k, Hq=4, Hkv=2, D=8, seed=0, lead=0, tail=0):
    """Random packed q [lead + sum(lens_q) + tail, Hq, D] and k/v [sum(lens_k) + tail, Hkv, D]
    with the cumulative offsets (sequence 0 starting at row `lead` of q)."""
    cq = np.concatenate([[0], np.cumsum(lens_q)]) + lead
    ck = np.concatenate([[0], np.cumsum(lens_k)])
    q = rnd((cq[-1] + tail, Hq, D), seed)
    k = rnd((ck[-1] + tail, Hkv, D), seed + 1)
    v = rnd((ck[-1] + tail, Hkv, D), seed + 2)
    return q, k, v, cq, ck


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_zero_query_is_mean_of_own_sequence(causal):
    # Q = 0: every visible score is 0, so O = mean of V over the row's visible keys of its
    # own sequence and LSE = log(count) -- fails on a wrong offset, a key leaking across a
    # sequence boundary, or a causal offset taken from the pack instead of the sequence
    lens_q, lens_k = [3, 5, 1, 4], [3, 7, 2, 4]
    q, k, v, cq, ck = packed(lens_q, lens_k, seed=4)
    q[:] = 0
    O, L = attention_varlen(q, k, v, cq, ck, 0.9, causal)
    G = 2
    for b in range(4):
        for i in range(lens_q[b]):
            n = visible_count(i, lens_q[b], lens_k[b], causal)
            r = cq[b] + i
            for h in range(4):
                np.testing.assert_allclose(O[r, h], v[ck[b]:ck[b] + n, h // G].mean(axis=0), atol=TOL)
                np.testing.assert_allclose(L[h, r], math.log(n), atol=TOL)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equal_lengths_is_batched_attention(causal):
    B, S = 3, 6
    q, k, v, cq, ck = packed([S] * B, [S] * B, seed=8)
    O, L = attention_varlen(q, k, v, cq, ck, 0.6, causal)
    Ob, Lb = attention(q.reshape(B, S, 4, 8), k.reshape(B, S, 2, 8), v.reshape(B, S, 2, 8), 0.6, causal)
    np.testing.assert_allclose(O, Ob.reshape(B * S, 4, 8), atol=TOL)
    np.testing.assert_allclose(L, Lb.transpose(1, 0, 2).reshape(4, B * S), atol=TOL)


def test_varlen_sequence_order_does_not_matter():
    # packing the same sequences in the opposite order moves their outputs with them
    lens = [4, 1, 6]
    q, k, v, cq, ck = packed(lens, lens, seed=13)
    O, L = attention_varlen(q, k, v, cq, ck, 0.5, True)
    order = [2, 1, 0]
    qs = np.concatenate([q[cq[b]:cq[b + 1]] for b in order])
    ks = np.concatenate([k[ck[b]:ck[b + 1]] for b in order])
    vs = np.concatenate([v[ck[b]:ck[b + 1]] for b in order])
    c2 = np.concatenate([[0], np.cumsum([lens[b] for b in order])])
    O2, L2 = attention_varlen(qs, ks, vs, c2, c2, 0.5, True)
    for n, b in enumerate(order):
        np.testing.assert_allclose(O2[c2[n]:c2[n + 1]], O[cq[b]:cq[b + 1]], atol=TOL)
        np.testing.assert_allclose(L2[:, c2[n]:c2[n + 1]], L[:, cq[b]:cq[b + 1]], atol=TOL)


def test_varlen_empty_single_key_and_uncovered_rows():
    # sequence 0: no keys (O = 0, LSE = -inf); 1: no queries; 2: one key (O = its V row,
    # LSE = its score); rows before the first and after the last sequence untouched
    lens_q, lens_k = [2, 0, 3], [0, 5, 1]
    q, k, v, cq, ck = packed(lens_q, lens_k, seed=21, lead=2, tail=3)
    O, L = attention_varlen(q, k, v, cq, ck, 0.7, False)
    assert np.all(O[cq[0]:cq[1]] == 0) and np.all(np.isneginf(L[:, cq[0]:cq[1]]))
    for r in range(cq[2], cq[3]):
        for h in range(4):
            np.testing.assert_allclose(O[r, h], v[ck[2], h // 2], atol=TOL)
            np.testing.assert_allclose(L[h, r], 0.7 * (q[r, h] @ k[ck[2], h // 2]), atol=TOL)
    for r in list(range(cq[0])) + list(range(cq[-1], q.shape[0])):
        assert np.all(O[r] == 0) and np.all(np.isneginf(L[:, r]))


def test_varlen_chunked_prefill_last_row_is_decode():
    # queries fewer than keys (a chunk appended to a cached prefix): with bottom-right
    # alignment the chunk's last row sees every key of its sequence, the first row
    # Sk - Sq + 1 of them
    lens_q, lens_k = [3, 2], [9, 5]
    q, k, v, cq, ck = packed(lens_q, lens_k, seed=30)
    O, L = attention_varlen(q, k, v, cq, ck, 0.4, True)
    for b in range(2):
        r = cq[b + 1] - 1
        Od, Ld = decode(q[None, r], k[None, ck[b]:ck[b + 1]], v[None, ck[b]:ck[b + 1]], 0.4)
        np.testing.assert_allclose(O[r], Od[0], atol=TOL)
        np.testing.assert_allclose(L[:, r], Ld[0], atol=TOL)
        n = lens_k[b] - lens_q[b] + 1
        Od, Ld = decode(q[None, cq[b]], k[None, ck[b]:ck[b] + n], v[None, ck[b]:ck[b] + n], 0.4)
        np.testing.assert_allclose(O[cq[b]], Od[0], atol=TOL)
        np.testing.assert_allclose(L[:, cq[b]], Ld[0], atol=TOL)


# ---- block-sparse attention: a 0/1 mask over (query block, key block) on top of the
#      dense rule (tiny blocks so the pins stay small)

def rand_mask(B, Hq, nq, nk, density, seed):
    return (np.random.default_rng(seed).random((B, Hq, nq, nk)) < density).astype(np.uint8)


@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_all_kept_is_dense(causal):
    q, k, v = qkv(B=2, Sq=10, Sk=10, Hq=4, Hkv=2, seed=51)
    m = np.ones((2, 4, 3, 3), np.uint8)
    O, L = attention_block_sparse(q, k, v, m, 0.3, causal, block=4)
    Od, Ld = attention(q, k, v, 0.3, causal)
    np.testing.assert_allclose(O, Od, atol=TOL)
    np.testing.assert_allclose(L, Ld, atol=TOL)


def test_block_sparse_lower_block_triangle_with_causal_is_causal():
    # blocks above the diagonal are causally invisible anyway
    q, k, v = qkv(B=1, Sq=12, Sk=12, Hq=2, Hkv=1, seed=52)
    m = np.tril(np.ones((3, 3), np.uint8))[None, None].repeat(2, axis=1)
    O, L = attention_block_sparse(q, k, v, m, 0.3, True, block=4)
    Od, Ld = attention(q, k, v, 0.3, True)
    np.testing.assert_allclose(O, Od, atol=TOL)
    np.testing.assert_allclose(L, Ld, atol=TOL)


def test_block_sparse_diagonal_blocks_are_independent_attentions():
    q, k, v = qkv(B=1, Sq=12, Sk=12, Hq=2, Hkv=2, seed=53)
    m = np.eye(3, dtype=np.uint8)[None, None].repeat(2, axis=1)
    O, L = attention_block_sparse(q, k, v, m, 0.5, False, block=4)
    for i in range(3):
        sl = slice(4 * i, 4 * i + 4)
        Ob, Lb = attention(q[:, sl], k[:, sl], v[:, sl], 0.5, False)
        np.testing.assert_allclose(O[:, sl], Ob, atol=TOL)
        np.testing.assert_allclose(L[:, :, sl], Lb, atol=TOL)


def test_block_sparse_equals_attention_over_the_gathered_keys():
    # non-causal: each query block attends exactly the concatenation of its kept key blocks
    B, Sq, Sk, Hq, Hkv, blk = 1, 11, 14, 4, 2, 4
    q, k, v = qkv(B=B, Sq=Sq, Sk=Sk, Hq=Hq, Hkv=Hkv, seed=54)
    m = rand_mask(B, Hq, 3, 4, 0.5, seed=9)
    O, L = attention_block_sparse(q, k, v, m, 0.4, False, block=blk)
    for h in range(Hq):
        for qi in range(3):
            keys = [j for ki in range(4) if m[0, h, qi, ki] for j in range(ki * blk, min(Sk, ki * blk + blk))]
            rows = slice(qi * blk, min(Sq, qi * blk + blk))
            if not keys:
                assert np.all(O[0, rows, h] == 0) and np.all(np.isneginf(L[0, h, rows]))
                continue
            kk = k[:, keys][:, :, [h // 2]]
            vv = v[:, keys][:, :, [h // 2]]
            Og, Lg = attention(q[:, rows][:, :, [h]], kk, vv, 0.4, False)
            np.testing.assert_allclose(O[0, rows, h], Og[0, :, 0], atol=TOL)
            np.testing.assert_allclose(L[0, h, rows], Lg[0, 0], atol=TOL)


@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_zero_query_is_mean_over_kept_visible_keys(causal):
    Sq, Sk, blk = 9, 13, 4
    q, k, v = qkv(B=1, Sq=Sq, Sk=Sk, Hq=2, Hkv=1, seed=55)
    q[:] = 0
    m = rand_mask(1, 2, 3, 4, 0.6, seed=4)
    O, L = attention_block_sparse(q, k, v, m, 1.0, causal, block=blk)
    for h in range(2):
        for i in range(Sq):
            keys = [j for j in range(Sk) if m[0, h, i // blk, j // blk] and (not causal or j <= i + Sk - Sq)]
            if not keys:
                assert np.all(O[0, i, h] == 0) and np.isneginf(L[0, h, i])
            else:
                np.testing.assert_allclose(O[0, i, h], v[0, keys, 0].mean(axis=0), atol=TOL)
                np.testing.assert_allclose(L[0, h, i], math.log(len(keys)), atol=TOL)


def test_block_sparse_rows_match_full():
    q, k, v = qkv(B=2, Sq=13, Sk=17, Hq=4, Hkv=2, seed=56)
    m = rand_mask(2, 4, 4, 5, 0.5, seed=5)
    O, L = attention_block_sparse(q, k, v, m, 0.3, True, block=4)
    rows = [0, 3, 4, 12]
    Or, Lr = attention_block_sparse_rows(q, k, v, m, 0.3, True, 1, 3, rows, block=4)
    np.testing.assert_allclose(Or, O[1, rows, 3], atol=TOL)
    np.testing.assert_allclose(Lr, L[1, 3, rows], atol=TOL)


@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_pair_count_by_brute_force(causal):
    Sq, Sk, blk = 10, 14, 4
    m = rand_mask(2, 3, 3, 4, 0.5, seed=6)
    n = 0
    for b in range(2):
        for h in range(3):
            for i in range(Sq):
                for j in range(Sk):
                    n += bool(m[b, h, i // blk, j // blk]) and (not causal or j <= i + Sk - Sq)
    assert block_sparse_pairs(Sq, Sk, m, causal, block=blk) == n
    ones = np.ones((1, 1, 3, 3), np.uint8)
    assert block_sparse_pairs(12, 12, ones, True, block=4) == 12 * 13 // 2
    assert block_sparse_pairs(12, 12, ones, False, block=4) == 144


def test_bench_block_sparse_flop_count_matches_the_oracle_count():
    from online_softmax_attention_sm_b200.workloads import block_sparse_flops
    for Sq, Sk, causal, seed in ((10, 14, True, 1), (13, 9, True, 2), (12, 12, False, 3), (7, 20, True, 4)):
        m = rand_mask(2, 3, -(-Sq // 4), -(-Sk // 4), 0.5, seed)
        assert block_sparse_flops(m, Sq, Sk, 8, causal, block=4) == 4 * 8 * block_sparse_pairs(Sq, Sk, m, causal,
                                                                                               block=4)


# ---- backward: gradients of L = sum(O * dO)

def loss(q, k, v, do, scale, causal):
    O, _ = attention(q, k, v, scale, causal)
    return float((O * do).sum())


@pytest.mark.parametrize("causal,Sq,Sk", [(False, 3, 4), (True, 4, 4), (True, 3, 5)])
def test_backward_matches_central_differences(causal, Sq, Sk):
    # brute force: every input element perturbed by +-eps, the loss re-evaluated
    q, k, v = qkv(B=1, Sq=Sq, Sk=Sk, Hq=2, Hkv=1, D=3, seed=71)
    do = rnd(q.shape, 72)
    dq, dk, dv = attention_backward(q, k, v, do, 0.7, causal)
    eps = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            old = x[idx]
            x[idx] = old + eps
            lp = loss(q, k, v, do, 0.7, causal)
            x[idx] = old - eps
            lm = loss(q, k, v, do, 0.7, causal)
            x[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7)


def test_backward_zero_query_dv_is_the_mean_of_do():
    # Q = 0: uniform weights over the visible keys, so dV_j = sum over rows i that see j
    # of dO_i / |V_i|
    Sq, Sk = 5, 5
    q, k, v = qkv(B=1, Sq=Sq, Sk=Sk, Hq=1, Hkv=1, D=4, seed=73)
    q[:] = 0
    do = rnd(q.shape, 74)
    _, _, dv = attention_backward(q, k, v, do, 1.0, True)
    want = np.zeros((Sk, 4))
    for i in range(Sq):
        n = visible_count(i, Sq, Sk, True)
        want[:n] += do[0, i, 0] / n
    np.testing.assert_allclose(dv[0, :, 0], want, atol=TOL)


def test_backward_equal_keys_give_zero_dq():
    # all keys equal: every score of a row is the same, so moving q changes nothing
    q, k, v = qkv(B=1, Sq=4, Sk=6, Hq=2, Hkv=2, D=5, seed=75)
    k[:] = k[:, :1]
    do = rnd(q.shape, 76)
    dq, _, _ = attention_backward(q, k, v, do, 0.9, False)
    np.testing.assert_allclose(dq, 0, atol=TOL)


def test_backward_gqa_is_mha_on_repeated_kv_summed():
    q, k, v = qkv(B=2, Sq=5, Sk=6, Hq=4, Hkv=2, D=3, seed=77)
    do = rnd(q.shape, 78)
    dq, dk, dv = attention_backward(q, k, v, do, 0.5, True)
    kr, vr = np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2)
    dq2, dk2, dv2 = attention_backward(q, kr, vr, do, 0.5, True)
    np.testing.assert_allclose(dq, dq2, atol=TOL)
    np.testing.assert_allclose(dk, dk2.reshape(2, 6, 2, 2, 3).sum(axis=3), atol=TOL)
    np.testing.assert_allclose(dv, dv2.reshape(2, 6, 2, 2, 3).sum(axis=3), atol=TOL)


def test_backward_rows_without_keys_contribute_nothing():
    # causal with Sq > Sk: the first Sq - Sk rows see no key
    q, k, v = qkv(B=1, Sq=6, Sk=3, Hq=1, Hkv=1, D=2, seed=79)
    do = rnd(q.shape, 80)
    dq, dk, dv = attention_backward(q, k, v, do, 0.8, True)
    assert np.all(dq[0, :3] == 0)
    do2 = do.copy()
    do2[0, :3] = 123.0                       # upstream gradient of those rows is irrelevant
    dq2, dk2, dv2 = attention_backward(q, k, v, do2, 0.8, True)
    np.testing.assert_allclose(dk2, dk, atol=TOL)
    np.testing.assert_allclose(dv2, dv, atol=TOL)


@pytest.mark.parametrize("causal,Sq,Sk", [(False, 7, 9), (True, 9, 9), (True, 6, 11), (True, 11, 6)])
def test_backward_rows_and_keys_match_the_full_backward(causal, Sq, Sk):
    # the sampled forms give the full backward's dQ rows and dK / dV keys, GQA included,
    # for rows that see no key (Sq > Sk) and keys that no row sees in full
    from oracle import attention_backward_keys, attention_backward_rows
    q, k, v = qkv(B=2, Sq=Sq, Sk=Sk, Hq=6, Hkv=2, D=5, seed=81)
    do = rnd(q.shape, 82)
    dq, dk, dv = attention_backward(q, k, v, do, 0.6, causal)
    rows = [0, Sq // 2, Sq - 1]
    keys = [0, Sk // 3, Sk - 2, Sk - 1]
    for b in range(2):
        for h in range(6):
            np.testing.assert_allclose(attention_backward_rows(q, k, v, do, 0.6, causal, b, h, rows),
                                       dq[b, rows, h], atol=TOL)
        for kvh in range(2):
            gk, gv = attention_backward_keys(q, k, v, do, 0.6, causal, b, kvh, keys)
            np.testing.assert_allclose(gk, dk[b, keys, kvh], atol=TOL)
            np.testing.assert_allclose(gv, dv[b, keys, kvh], atol=TOL)


def test_backward_rows_and_keys_match_central_differences():
    # brute force on a tiny causal GQA case, independent of the full backward
    from oracle import attention_backward_keys, attention_backward_rows
    q, k, v = qkv(B=1, Sq=4, Sk=5, Hq=2, Hkv=1, D=3, seed=83)
    do = rnd(q.shape, 84)
    eps = 1e-6

    def num_grad(x, idx):
        old = x[idx]
        x[idx] = old + eps
        lp = loss(q, k, v, do, 0.7, True)
        x[idx] = old - eps
        lm = loss(q, k, v, do, 0.7, True)
        x[idx] = old
        return (lp - lm) / (2 * eps)

    dq = attention_backward_rows(q, k, v, do, 0.7, True, 0, 1, [2, 3])
    for r, i in enumerate([2, 3]):
        for d in range(3):
            assert abs(dq[r, d] - num_grad(q, (0, i, 1, d))) < 1e-7
    dk, dv = attention_backward_keys(q, k, v, do, 0.7, True, 0, 0, [1, 4])
    for r, j in enumerate([1, 4]):
        for d in range(3):
            assert abs(dk[r, d] - num_grad(k, (0, j, 0, d))) < 1e-7
            assert abs(dv[r, d] - num_grad(v, (0, j, 0, d))) < 1e-7


# ---- FP8 (e4m3) inputs

def test_decode_e4m3_known_codes():
    from oracle import decode_e4m3
    table = {0x00: 0.0, 0x38: 1.0, 0xB8: -1.0, 0x40: 2.0, 0x3C: 1.5, 0x7E: 448.0, 0xFE: -448.0,
             0x08: 2.0 ** -6, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x30: 0.5, 0x77: 240.0}
    for code, val in table.items():
        assert decode_e4m3([code])[0] == val, hex(code)
    assert np.isnan(decode_e4m3([0x7F])[0]) and np.isnan(decode_e4m3([0xFF])[0])


def test_decode_e4m3_matches_torch_float8():
    # every code against the library's own float8_e4m3fn -> float conversion
    import torch
    from oracle import decode_e4m3
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = decode_e4m3(codes)
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib))
    np.testing.assert_array_equal(ours[~np.isnan(ours)], lib[~np.isnan(lib)])


def test_attention_fp8_is_attention_of_the_dequantised_inputs():
    from oracle import attention_fp8, decode_e4m3
    rng = np.random.default_rng(3)
    q8, k8, v8 = (rng.integers(0, 0x7E, size=s, dtype=np.uint8) for s in ((1, 5, 2, 4), (1, 7, 1, 4), (1, 7, 1, 4)))
    O, L = attention_fp8(q8, k8, v8, 0.01, 0.02, 0.5, 0.7, True)
    Od, Ld = attention(decode_e4m3(q8) * 0.01, decode_e4m3(k8) * 0.02, decode_e4m3(v8) * 0.5, 0.7, True)
    np.testing.assert_allclose(O, Od, atol=TOL)
    np.testing.assert_allclose(L, Ld, atol=TOL)


# ---- packed queries against a paged K/V cache

def test_paged_prefill_is_varlen_over_gathered_keys():
    from oracle import attention_paged_prefill
    # two sequences; queries are chunks at the end of their keys (chunked prefill)
    lens_q, lens_k, page = [3, 5], [9, 6], 4
    rng = np.random.default_rng(0)
    q = rng.standard_normal((8, 4, 3))
    k = rng.standard_normal((15, 2, 3))
    v = rng.standard_normal((15, 2, 3))
    cq, ck = np.array([0, 3, 8]), np.array([0, 9, 15])
    O, L = attention_varlen(q, k, v, cq, ck, 0.6, True)
    # pages of 4 keys, shuffled: sequence 0 -> 3 pages, sequence 1 -> 2 pages
    perm = rng.permutation(6)
    kc, vc = np.zeros((6, page, 2, 3)), np.zeros((6, page, 2, 3))
    table = np.full((2, 3), 0)
    for b, (k0, n) in enumerate(((0, 9), (9, 6))):
        for i in range(-(-n // page)):
            slot = perm[3 * b + i] if b == 0 else perm[3 + i]
            rows = range(k0 + i * page, min(k0 + n, k0 + (i + 1) * page))
            kc[slot, :len(rows)], vc[slot, :len(rows)] = k[list(rows)], v[list(rows)]
            table[b, i] = slot
    Op, Lp = attention_paged_prefill(q, kc, vc, cq, table, np.array(lens_k), 0.6, True)
    np.testing.assert_allclose(Op, O, atol=TOL)
    np.testing.assert_allclose(Lp, L, atol=TOL)


def test_paged_prefill_lengths_clamp_and_empty():
    from oracle import attention_paged_prefill
    rng = np.random.default_rng(1)
    q = rng.standard_normal((4, 2, 3))
    kc, vc = rng.standard_normal((3, 4, 1, 3)), rng.standard_normal((3, 4, 1, 3))
    table = np.array([[2, 0], [1, 1]])
    cq = np.array([0, 2, 4])
    O, L = attention_paged_prefill(q, kc, vc, cq, table, np.array([100, 0]), 0.5, False)
    # sequence 0 clamps to its 8 keys: pages 2 then 0
    keys = np.concatenate([kc[2], kc[0]])[None]
    vals = np.concatenate([vc[2], vc[0]])[None]
    Od, Ld = attention(q[None, :2], keys, vals, 0.5, False)
    np.testing.assert_allclose(O[:2], Od[0], atol=TOL)
    np.testing.assert_allclose(L[:, :2], Ld[0], atol=TOL)
    assert np.all(O[2:] == 0) and np.all(np.isneginf(L[:, 2:]))           # no keys


def test_e4m3_quantisation_round_trip_fixes_the_descale_direction():
    # the input recipe's per-tensor quantisation, then decode_e4m3(codes) * descale: every value
    # comes back within half an e4m3 step (2^-4 relative in the normal range, 2^-10 * descale
    # below it); dividing by the descale instead, or forgetting it, misses by orders of magnitude
    import torch
    from oracle import decode_e4m3
    from online_softmax_attention_sm_b200.inputs import quantize_e4m3
    x = torch.randn(4096, generator=torch.Generator().manual_seed(5), dtype=torch.float32) * 3.0
    codes, d = quantize_e4m3(x)
    back = decode_e4m3(codes.numpy()) * d
    xs = x.double().numpy()
    allowed = np.maximum(2.0 ** -4 * np.abs(xs), 2.0 ** -10 * d)
    assert np.all(np.abs(back - xs) <= allowed * (1 + 1e-12))
    assert np.abs(back).max() == pytest.approx(np.abs(xs).max(), rel=1e-6)   # amax maps to 448 exactly


def test_attention_fp8_closed_forms_fix_each_descale():
    from oracle import attention_fp8, decode_e4m3
    rng = np.random.default_rng(11)
    qd, kd, vd, scale = 0.03, 0.2, 1.7, 0.8
    k8 = rng.integers(0x20, 0x60, size=(1, 6, 1, 4), dtype=np.uint8)
    v8 = rng.integers(0x20, 0x60, size=(1, 6, 1, 4), dtype=np.uint8)
    vals = (decode_e4m3(v8) * vd)[0, :, 0]                       # V as the caller means it
    # Q = 0 (code 0): uniform weights, O = the mean of the dequantised V over the visible keys
    q0 = np.zeros((1, 6, 2, 4), dtype=np.uint8)
    O, L = attention_fp8(q0, k8, v8, qd, kd, vd, scale, causal=True)
    for i in range(6):
        np.testing.assert_allclose(O[0, i, 1], vals[: i + 1].mean(axis=0), atol=1e-12)
        assert L[0, 1, i] == pytest.approx(math.log(i + 1), abs=1e-12)
    # a single key: O = its V row, LSE = scale * (q qd) . (k kd), summed by hand
    q8 = rng.integers(0x20, 0x60, size=(1, 3, 1, 4), dtype=np.uint8)
    O, L = attention_fp8(q8, k8[:, :1], v8[:, :1], qd, kd, vd, scale, causal=False)
    qv, kv = decode_e4m3(q8)[0, :, 0], decode_e4m3(k8)[0, 0, 0]
    for i in range(3):
        dot = sum(float(qv[i, d]) * qd * float(kv[d]) * kd for d in range(4))
        assert L[0, 0, i] == pytest.approx(scale * dot, abs=1e-12)
        np.testing.assert_allclose(O[0, i, 0], vals[0], atol=1e-12)


def test_attention_fp8_approximates_attention_of_the_unquantised_inputs():
    # quantise float inputs with the recipe, run the FP8 oracle, compare with attention of the
    # original floats: close (quantisation error only), which fails if any descale is applied
    # the wrong way round or to the wrong tensor
    import torch
    from oracle import attention_fp8
    from online_softmax_attention_sm_b200.inputs import make_qkv_fp8, make_qkv
    args = (1, 40, 40, 2, 1, 16)
    q8, k8, v8, qd, kd, vd = make_qkv_fp8(*args, seed=9, input_scale=0.7)
    q, k, v = (t.double().numpy() for t in make_qkv(*args, "fp32", 9, 0.7))
    assert not (qd == kd or kd == vd or qd == vd)
    O, L = attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), qd, kd, vd, 0.25, True)
    Oe, Le = attention(q, k, v, 0.25, True)
    assert np.abs(O - Oe).max() < 0.1 and np.abs(L - Le).max() < 0.1
    for wrong in ((1 / qd, kd, vd), (qd, kd, 1 / vd), (vd, kd, qd), (qd, vd, kd)):
        Ow, Lw = attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), *wrong, 0.25, True)
        assert np.abs(Ow - Oe).max() > 0.1 or np.abs(Lw - Le).max() > 0.1
