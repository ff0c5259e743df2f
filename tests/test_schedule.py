"""Host-side check of the prefill's unit enumeration (a mirror of the kernel's fwd_unit and
of the host's choice of group and band, plan_units, including its short-sequence branch):
every (batch, head, query block) is produced exactly once, heads map to their KV head, and
the order keeps the longest units first within each band -- across every pair when the
short-sequence branch applies."""
import math

import pytest


def choose(B, Sq, Sk, Hq, Hkv, D, ncta=148, l2=126 * 2 ** 20):
    n_qblk = (Sq + 255) // 256
    n_units = B * Hq * n_qblk
    ncta = min(n_units, ncta)
    G, n_bk = Hq // Hkv, B * Hkv
    gmax = max(1, min(n_bk, int((l2 // 2) / (2.0 * Sk * D * 2))))
    best = (1e30, 1, 1)
    for g in range(1, gmax + 1):
        band = (ncta + g * G - 1) // (g * G)
        waste = (band * g * G % ncta) / ncta
        if waste < best[0] - 1e-9:
            best = (waste, g, band)
    kg, band = best[1], best[2]
    if band >= n_qblk and n_qblk > 4:
        # short sequences: bands of one query block over every (batch, KV head) pair
        return n_bk, 1
    return kg, min(band, n_qblk)


def unit(u, B, Sq, Hq, Hkv, kv_group, band):
    n_qblk = (Sq + 255) // 256
    G, n_bk = Hq // Hkv, B * Hkv
    per_band = band * B * Hq
    bi = u // per_band
    bs = min(band, n_qblk - bi * band)
    r = u - bi * per_band
    full_grp = kv_group * G * bs
    g = r // full_grp
    gsize = min(kv_group, n_bk - g * kv_group)
    rr = r - g * full_grp
    qb = n_qblk - 1 - (bi * band + rr // (gsize * G))
    rem = rr % (gsize * G)
    bk = g * kv_group + rem // G
    b, kvh = divmod(bk, Hkv)
    return b, kvh * G + rem % G, qb, bi


@pytest.mark.parametrize("shape", [(1, 32768, 32768, 32, 8, 128), (2, 4096, 4096, 8, 8, 128), (1, 2048, 2048, 16, 16, 64),
                                   (1, 128, 128, 2, 2, 64), (3, 1000, 777, 14, 2, 64), (2, 513, 1000, 4, 1, 128),
                                   (5, 300, 300, 7, 7, 64), (1, 65536, 65536, 8, 1, 128), (1, 1, 1, 1, 1, 64)])
def test_unit_order_is_a_bijection(shape):
    B, Sq, Sk, Hq, Hkv, D = shape
    kg, band = choose(B, Sq, Sk, Hq, Hkv, D)
    n_qblk = (Sq + 255) // 256
    seen = set()
    last_band, band_max_qb = -1, None
    for u in range(B * Hq * n_qblk):
        b, h, qb, bi = unit(u, B, Sq, Hq, Hkv, kg, band)
        assert 0 <= b < B and 0 <= h < Hq and 0 <= qb < n_qblk
        seen.add((b, h, qb))
        assert bi >= last_band                      # bands in order: longest blocks first
        last_band = bi
    assert len(seen) == B * Hq * n_qblk


def test_long_gqa_workload_choice():
    # 32768 tokens, 8 KV heads of 16.8 MB K+V each: one KV head per group, 37-block bands
    assert choose(1, 32768, 32768, 32, 8, 128) == (1, 37)


def test_short_sequences_go_longest_first_across_all_pairs():
    # 2048 tokens, 16 batches: one band would hold all 8 query blocks, so the host takes
    # bands of one query block over all (batch, KV head) pairs
    B, Sq, Sk, Hq, Hkv, D = 16, 2048, 2048, 8, 2, 128
    kg, band = choose(B, Sq, Sk, Hq, Hkv, D)
    assert (kg, band) == (B * Hkv, 1)
    n_qblk = (Sq + 255) // 256
    qbs = [unit(u, B, Sq, Hq, Hkv, kg, band)[2] for u in range(B * Hq * n_qblk)]
    assert qbs == sorted(qbs, reverse=True)          # strictly longest query blocks first
    assert len({(b, h, qb) for b, h, qb, _ in (unit(u, B, Sq, Hq, Hkv, kg, band)
                                                for u in range(B * Hq * n_qblk))}) == B * Hq * n_qblk
