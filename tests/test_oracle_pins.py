"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: a closed form,
an explicit numpy float64 matrix route written here, an invariant of softmax
attention, or brute force on tiny inputs. The pages print no worked example for
this computation (the one figure they do print, the size of a dense score
matrix, is pinned by the golden test), so these are the pins.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from mla_flash_attention_attn_b200 import workloads as W

DK, DV = 576, 512
NEG = np.float16(-np.inf)


def rand_f16(rng, shape, std=1.0):
    return (rng.standard_normal(shape) * std).astype(np.float16)


def brute_force(q, k, mask, scale):
    """softmax(scale * Q K^T + mask) V with explicit float64 matrices.

    q [n_q][H][576] f16, k [n][576] f16, mask [n_q][n] f16 or None."""
    qd = q.astype(np.float64)
    kd = k.astype(np.float64)
    n_q, H, _ = q.shape
    out = np.zeros((n_q, H, DV))
    for t in range(n_q):
        S = scale * (qd[t] @ kd.T)  # [H][n]
        if mask is not None:
            S = S + mask[t].astype(np.float64)[None, :]
        mx = S.max(axis=1, keepdims=True)
        P = np.where(np.isneginf(S), 0.0, np.exp(S - np.where(np.isneginf(mx), 0.0, mx)))
        den = P.sum(axis=1, keepdims=True)
        with np.errstate(invalid="ignore", divide="ignore"):
            O = np.where(den > 0, (P @ kd[:, :DV]) / np.where(den > 0, den, 1.0), 0.0)
        out[t] = O
    return out.reshape(n_q * H, DV)


def test_half_conversion_matches_numpy_on_all_finite_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits[::97]])
    r = ref[::97]
    fin = np.isfinite(r)
    assert np.array_equal(got[fin], r[fin])
    assert oracle.half_to_double(0xFC00) == -math.inf
    assert oracle.half_to_double(0x7C00) == math.inf
    assert oracle.half_to_double(0x0001) == 2.0 ** -24


def test_single_key_gives_its_value_row_exactly():
    rng = np.random.default_rng(1)
    q = rand_f16(rng, (2, 3, DK))
    k = rand_f16(rng, (1, DK))
    for mask in (None, np.array([[1.5], [-7.0]], np.float16)):
        out = oracle.attention(q, k, mask=mask, scale=0.3)
        expect = np.broadcast_to(k[0, :DV].astype(np.float64), out.shape)
        assert np.array_equal(out, expect)


def test_zero_query_gives_mean_of_kept_values():
    rng = np.random.default_rng(2)
    n = 37
    q = np.zeros((1, 4, DK), np.float16)
    k = rand_f16(rng, (n, DK))
    keep = rng.random(n) < 0.6
    keep[0] = True
    mask = np.where(keep, np.float16(0), NEG).astype(np.float16)[None]
    out = oracle.attention(q, k, mask=mask, scale=1.0 / math.sqrt(192))
    mean = k[keep, :DV].astype(np.float64).mean(axis=0)
    np.testing.assert_allclose(out, np.broadcast_to(mean, out.shape), rtol=0, atol=1e-14)


def test_two_key_closed_form_and_mask_is_added_after_scaling():
    # Q = e_0 so the dot with key j is k[j][0]; scores s_j = scale*k_j0 + m_j.
    q = np.zeros((1, 1, DK), np.float16)
    q[0, 0, 0] = 1.0
    k = np.zeros((2, DK), np.float16)
    k[0, 0], k[1, 0] = 2.0, -1.0
    k[0, 1:DV] = 0.25
    k[1, 1:DV] = -0.5
    k[:, DV:] = 3.0  # rope columns take part in the dot product only through c=0 here
    scale = 0.5
    m = np.array([[0.75, 2.0]], np.float16)
    out = oracle.attention(q, k, mask=m, scale=scale)[0]
    s0 = scale * 2.0 + 0.75
    s1 = scale * -1.0 + 2.0
    delta = s1 - s0
    v0, v1 = k[0, :DV].astype(np.float64), k[1, :DV].astype(np.float64)
    expect = (v0 + math.exp(delta) * v1) / (1.0 + math.exp(delta))
    np.testing.assert_allclose(out, expect, rtol=1e-15, atol=1e-15)


def test_rope_columns_enter_the_score_but_not_the_value():
    # Q nonzero only on a rope column: the score must see it.
    q = np.zeros((1, 1, DK), np.float16)
    q[0, 0, 540] = 1.0
    k = np.zeros((2, DK), np.float16)
    k[0, 540] = 4.0
    k[0, :DV] = 1.0
    k[1, :DV] = -1.0
    out = oracle.attention(q, k, scale=1.0)[0]
    w1 = 1.0 / (1.0 + math.exp(4.0))
    expect = (1.0 - w1) * 1.0 + w1 * -1.0
    np.testing.assert_allclose(out, expect, rtol=1e-14)


@pytest.mark.parametrize("n_q,H,n", [(1, 1, 1), (1, 2, 5), (3, 2, 8), (2, 1, 7)])
def test_brute_force_tiny(n_q, H, n):
    rng = np.random.default_rng(100 + n_q * 10 + n)
    q = rand_f16(rng, (n_q, H, DK))
    k = rand_f16(rng, (n, DK))
    mask = rand_f16(rng, (n_q, n), std=2.0)
    mask[rng.random((n_q, n)) < 0.3] = NEG
    scale = 1.0 / math.sqrt(192)
    got = oracle.attention(q, k, mask=mask, scale=scale)
    np.testing.assert_allclose(got, brute_force(q, k, mask, scale), rtol=1e-12, atol=1e-13)


def test_brute_force_per_token_mask_rows_and_heads_distinct():
    # Distinct masks per token and distinct queries per head catch transposed indices.
    rng = np.random.default_rng(7)
    q = rand_f16(rng, (4, 3, DK))
    k = rand_f16(rng, (6, DK))
    mask = np.zeros((4, 6), np.float16)
    for t in range(4):
        mask[t, t + 1:] = NEG  # causal-like, different per token
    got = oracle.attention(q, k, mask=mask, scale=0.1)
    np.testing.assert_allclose(got, brute_force(q, k, mask, 0.1), rtol=1e-12, atol=1e-13)


def test_shift_invariance_of_mask():
    rng = np.random.default_rng(3)
    q = rand_f16(rng, (2, 2, DK))
    k = rand_f16(rng, (40, DK))
    mask = np.zeros((2, 40), np.float16)
    mask[:, 30:] = NEG
    base = oracle.attention(q, k, mask=mask, scale=0.07)
    shifted = np.where(np.isneginf(mask), mask, mask + np.float16(6.0)).astype(np.float16)
    np.testing.assert_allclose(oracle.attention(q, k, mask=shifted, scale=0.07), base,
                               rtol=1e-13, atol=1e-14)


def test_masked_garbage_rows_contribute_nothing_bit_identical():
    rng = np.random.default_rng(4)
    q = rand_f16(rng, (1, 3, DK))
    k = rand_f16(rng, (20, DK))
    mask = np.zeros((1, 20), np.float16)
    base = oracle.attention(q, k, mask=mask, scale=0.05)
    garbage = np.full((9, DK), np.float16(60000.0))
    garbage[::2] = np.float16(-60000.0)
    k2 = np.concatenate([k, garbage])
    mask2 = np.concatenate([mask, np.full((1, 9), NEG, np.float16)], axis=1)
    assert np.array_equal(oracle.attention(q, k2, mask=mask2, scale=0.05), base)


def test_fully_masked_row_is_zero():
    rng = np.random.default_rng(5)
    q = rand_f16(rng, (2, 2, DK))
    k = rand_f16(rng, (10, DK))
    mask = np.zeros((2, 10), np.float16)
    mask[1, :] = NEG
    out = oracle.attention(q, k, mask=mask, scale=0.1).reshape(2, 2, DV)
    assert np.all(out[1] == 0.0)
    assert np.all(np.abs(out[0]) > 0.0)


def test_permutation_invariance():
    rng = np.random.default_rng(6)
    q = rand_f16(rng, (2, 2, DK))
    k = rand_f16(rng, (33, DK))
    mask = rand_f16(rng, (2, 33))
    mask[:, ::5] = NEG
    perm = rng.permutation(33)
    a = oracle.attention(q, k, mask=mask, scale=0.06)
    b = oracle.attention(q, k[perm], mask=mask[:, perm], scale=0.06)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("tile", [1, 7, 64, 1000])
def test_online_matches_two_pass(tile):
    rng = np.random.default_rng(8)
    n = 150
    q = rand_f16(rng, (2, 2, DK))
    k = rand_f16(rng, (n, DK))
    mask = np.zeros((2, n), np.float16)
    mask[0, :40] = NEG  # first tiles fully masked for one row
    mask[1, 100:] = NEG
    a = oracle.attention(q, k, mask=mask, scale=0.09)
    b = oracle.attention_online(q, k, mask=mask, scale=0.09, tile=tile)
    np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-14)


def test_online_with_growing_scores_has_no_positional_bias():
    # Scores increase along the sequence, so the running max grows every tile: a broken
    # rescale would bias the late keys (the failure mode the article warns about).
    q = np.zeros((1, 1, DK), np.float16)
    q[0, 0, 0] = 1.0
    n = 64
    k = np.zeros((n, DK), np.float16)
    k[:, 0] = np.linspace(-8, 8, n).astype(np.float16)
    k[:, 1] = np.arange(n).astype(np.float16)
    a = oracle.attention(q, k, scale=1.0)
    b = oracle.attention_online(q, k, scale=1.0, tile=3)
    np.testing.assert_allclose(b, a, rtol=1e-12)
    np.testing.assert_allclose(a, brute_force(q, k, None, 1.0), rtol=1e-12)


@pytest.mark.parametrize("bounds", [[0, 50], [0, 1, 50], [0, 13, 13, 40, 50], [0, 20, 30, 49, 50]])
def test_split_combine_matches_unsplit(bounds):
    rng = np.random.default_rng(9)
    q = rand_f16(rng, (1, 3, DK))
    k = rand_f16(rng, (50, DK))
    mask = np.zeros((1, 50), np.float16)
    mask[0, 13:40] = NEG  # some parts fully masked (l_s = 0 parts are skipped)
    a = oracle.attention(q, k, mask=mask, scale=0.08)
    b = oracle.attention_split(q, k, mask=mask, scale=0.08, bounds=bounds)
    np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-14)


def test_rows_subset_matches_full():
    rng = np.random.default_rng(10)
    q = rand_f16(rng, (3, 4, DK))
    k = rand_f16(rng, (12, DK))
    full = oracle.attention(q, k, scale=0.1)
    rows = np.array([11, 0, 5], np.int32)
    assert np.array_equal(oracle.attention(q, k, scale=0.1, rows=rows), full[rows])


def test_compaction_brute_force_all_16_cell_masks():
    pats = np.arange(1 << 16, dtype=np.uint32)
    bits = ((pats[:, None] >> np.arange(16, dtype=np.uint32)[None, :]) & 1).astype(bool)
    for i in range(0, 1 << 16, 1):
        keep = bits[i]
        row = np.where(keep, np.float16(0), NEG).astype(np.float16)
        got = oracle.compact(row)
        assert np.array_equal(got, np.nonzero(keep)[0].astype(np.int32)), i


def test_compaction_keep_rule_only_minus_inf_dropped():
    row = np.array([0, -np.inf, -60000.0, np.inf, -0.0, 1e-7, -np.inf], np.float16)
    assert oracle.compact(row).tolist() == [0, 2, 3, 4, 5]
    row2 = np.full(1000, NEG, np.float16)
    assert len(oracle.compact(row2)) == 0


def test_compaction_random_long_rows_equal_numpy_filter():
    rng = np.random.default_rng(11)
    for n in (1, 31, 32, 33, 1023, 4097):
        keep = rng.random(n) < 0.3
        row = np.where(keep, rng.standard_normal(n), -np.inf).astype(np.float16)
        assert np.array_equal(oracle.compact(row), np.nonzero(keep)[0].astype(np.int32))


def test_q8_0_dequant_hand_built_blocks():
    n = 2
    d = np.ones((n, 18), np.float16)
    d[1] = np.float16(0.5)
    qv = np.zeros((n, 18, 32), np.int8)
    ramp = np.arange(-16, 16, dtype=np.int8)
    qv[0] = ramp[None, :]
    qv[1] = np.int8(-127)
    qv[1, 17, 31] = 127
    rows = W.q8_0_pack(d, qv)
    assert rows.shape == (2, 612)
    deq = oracle.dequant_q8_0(rows)
    assert np.array_equal(deq[0], np.tile(ramp.astype(np.float64), 18))
    expect1 = np.full(DK, -63.5)
    expect1[-1] = 63.5
    assert np.array_equal(deq[1], expect1)


def test_q8_0_attention_equals_f16_attention_on_exactly_representable_values():
    # d = 1/64 (a power of two) and |q| <= 127: d*q is exact in f16, so the q8_0 path must
    # equal the f16 path on the same values bit for bit.
    rng = np.random.default_rng(12)
    n = 45
    qv = rng.integers(-127, 128, size=(n, 18, 32)).astype(np.int8)
    d = np.full((n, 18), np.float16(1.0 / 64))
    rows = W.q8_0_pack(d, qv)
    kf16 = (qv.reshape(n, DK).astype(np.float32) / 64.0).astype(np.float16)
    q = rand_f16(rng, (1, 4, DK))
    mask = np.zeros((1, n), np.float16)
    mask[0, 7] = NEG
    a = oracle.attention(q, rows, kv_type=oracle.KV_Q8_0, mask=mask, scale=0.05)
    b = oracle.attention(q, kf16, kv_type=oracle.KV_F16, mask=mask, scale=0.05)
    assert np.array_equal(a, b)


def test_sparse_index_path_equals_dense_masked_path():
    rng = np.random.default_rng(13)
    n = 300
    q = rand_f16(rng, (1, 3, DK))
    k = rand_f16(rng, (n, DK))
    keep = rng.random(n) < 0.2
    mask = np.where(keep, np.float16(0), NEG).astype(np.float16)[None]
    idx = np.nonzero(keep)[0].astype(np.int32)
    dense = oracle.attention(q, k, mask=mask, scale=0.07)
    sparse = oracle.attention(q, k, mask=mask, scale=0.07, idx=idx)
    np.testing.assert_allclose(sparse, dense, rtol=1e-12, atol=1e-14)


def test_oracle_rejects_out_of_range_index():
    q = np.zeros((1, 1, DK), np.float16)
    k = np.zeros((4, DK), np.float16)
    with pytest.raises(ValueError):
        oracle.attention(q, k, idx=np.array([0, 4], np.int32))


def test_planted_mistakes_are_caught():
    """The checks above must fail on plausible oracle mistakes; emulate three of them on
    the CPU in numpy (wrong V columns, mask scaled, rope dropped) and confirm that the
    brute-force pin separates each from the oracle's answer."""
    rng = np.random.default_rng(14)
    q = rand_f16(rng, (2, 2, DK))
    k = rand_f16(rng, (9, DK))
    mask = rand_f16(rng, (2, 9), std=3.0)
    scale = 0.2
    ref = oracle.attention(q, k, mask=mask, scale=scale)

    def route(qq, kk, vv, mm):
        S = scale * np.einsum("thc,nc->thn", qq.astype(np.float64), kk.astype(np.float64))
        S = S + mm
        P = np.exp(S - S.max(-1, keepdims=True))
        P /= P.sum(-1, keepdims=True)
        return np.einsum("thn,nd->thd", P, vv.astype(np.float64)).reshape(-1, DV)

    m64 = mask.astype(np.float64)[:, None, :]
    good = route(q, k, k[:, :DV], m64)
    np.testing.assert_allclose(ref, good, rtol=1e-12, atol=1e-13)
    wrong_v = route(q, k, k[:, DK - DV:], m64)
    scaled_mask = route(q, k, k[:, :DV], scale * m64)
    q_norope = q.copy()
    q_norope[..., DV:] = 0
    no_rope = route(q_norope, k, k[:, :DV], m64)
    for bad in (wrong_v, scaled_mask, no_rope):
        assert np.max(np.abs(bad - ref)) > 1e-3


# ---- value up-projection W_UV (oracle.project), pinned to other computations --------

def _proj_inputs(seed, n_rows=12, n_head=4, proj_dim=128):
    rng = np.random.default_rng(seed)
    o = rng.standard_normal((n_rows, oracle.DV))
    heads = rng.integers(0, n_head, n_rows).astype(np.int32)
    wv = (rng.standard_normal((n_head, oracle.DV, proj_dim)) * 0.05).astype(np.float16)
    return o, heads, wv


def test_project_one_hot_weights_select_columns_exactly():
    # wv[h][d][n] = 1 where d = sel[h][n]: each output is one input column, exactly
    rng = np.random.default_rng(51)
    n_head, proj_dim, n_rows = 3, 128, 10
    o = rng.standard_normal((n_rows, oracle.DV))
    heads = rng.integers(0, n_head, n_rows).astype(np.int32)
    sel = np.stack([rng.permutation(oracle.DV)[:proj_dim] for _ in range(n_head)])
    wv = np.zeros((n_head, oracle.DV, proj_dim), dtype=np.float16)
    for h in range(n_head):
        wv[h, sel[h], np.arange(proj_dim)] = 1.0
    got = oracle.project(o, heads, wv)
    want = np.stack([o[r, sel[heads[r]]] for r in range(n_rows)])
    assert np.array_equal(got, want)


def test_project_weights_of_each_head_are_its_own():
    # head h scales its selector by 2^h: a row projected with another head's matrix
    # would come out with the wrong power of two
    rng = np.random.default_rng(52)
    n_head, n_rows = 4, 16
    o = rng.standard_normal((n_rows, oracle.DV))
    heads = (np.arange(n_rows) % n_head).astype(np.int32)
    wv = np.zeros((n_head, oracle.DV, 128), dtype=np.float16)
    for h in range(n_head):
        wv[h, np.arange(128), np.arange(128)] = 2.0 ** h
    got = oracle.project(o, heads, wv)
    want = np.stack([o[r, :128] * 2.0 ** heads[r] for r in range(n_rows)])
    assert np.array_equal(got, want)


def test_project_scales_exactly_with_a_power_of_two():
    o, heads, wv = _proj_inputs(53)
    a = oracle.project(o, heads, wv)
    b = oracle.project(o, heads, (wv.astype(np.float32) * 4).astype(np.float16))
    assert np.array_equal(b, 4 * a)


def test_project_matches_an_independent_contraction():
    # numpy's fp64 contraction over the exactly converted f16 weights; only the
    # summation order differs
    o, heads, wv = _proj_inputs(54)
    want = np.einsum("rd,rdn->rn", o, wv.astype(np.float64)[heads])
    got = oracle.project(o, heads, wv)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_project_rejects_bad_heads():
    o, heads, wv = _proj_inputs(55)
    heads[3] = 4  # n_head is 4
    with pytest.raises(ValueError):
        oracle.project(o, heads, wv)


# ---- attention variants: softcap, ALiBi, sinks (oracle.attention_variants) -----------

def brute_force_variants(q, k, mask, scale, softcap=0.0, slopes=None, pos0=0, sinks=None):
    """The variants' definitions with explicit float64 numpy matrices (no oracle code)."""
    qd = q.astype(np.float64)
    kd = k.astype(np.float64)
    n_q, H, _ = q.shape
    n = k.shape[0]
    out = np.zeros((n_q, H, DV))
    for t in range(n_q):
        S = scale * (qd[t] @ kd.T)  # [H][n]
        if softcap > 0:
            S = softcap * np.tanh(S / softcap)
        if mask is not None:
            S = S + mask[t].astype(np.float64)[None, :]
        if slopes is not None:
            S = S + np.asarray(slopes, np.float64)[:, None] * (np.arange(n)[None, :] - (pos0 + t))
        M = S.max(axis=1)
        if sinks is not None:
            M = np.maximum(M, np.asarray(sinks, np.float64))
        for h in range(H):
            if np.isneginf(M[h]):
                continue
            p = np.where(np.isneginf(S[h]), 0.0, np.exp(S[h] - M[h]))
            den = p.sum() + (np.exp(sinks[h] - M[h]) if sinks is not None else 0.0)
            out[t, h] = (p @ kd[:, :DV]) / den
    return out.reshape(n_q * H, DV)


def _variant_inputs(seed, n_q=2, H=4, n=37, masked=True):
    rng = np.random.default_rng(seed)
    q = rand_f16(rng, (n_q, H, DK))
    k = rand_f16(rng, (n, DK))
    mask = None
    if masked:
        mask = rand_f16(rng, (n_q, n), std=0.5)
        mask[:, rng.choice(n, 5, replace=False)] = NEG
    return q, k, mask


def test_softcap_matches_brute_force():
    q, k, mask = _variant_inputs(61)
    got = oracle.attention_variants(q, k, mask=mask, scale=0.125, softcap=2.5)
    want = brute_force_variants(q, k, mask, 0.125, softcap=2.5)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12)


def test_softcap_with_a_huge_cap_is_plain_attention():
    q, k, mask = _variant_inputs(62)
    got = oracle.attention_variants(q, k, mask=mask, scale=0.125, softcap=1e7)
    want = brute_force(q, k, mask, 0.125).reshape(-1, DV)
    assert np.allclose(got, want, rtol=1e-9, atol=1e-12)


def test_alibi_matches_brute_force_and_is_shift_invariant():
    q, k, mask = _variant_inputs(63)
    slopes = np.array([0.5, 0.25, 0.125, 0.0625])
    got = oracle.attention_variants(q, k, mask=mask, scale=0.125, slopes=slopes, pos0=36)
    want = brute_force_variants(q, k, mask, 0.125, slopes=slopes, pos0=36)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12)
    # a per-row constant in the bias does not change a softmax
    shifted = oracle.attention_variants(q, k, mask=mask, scale=0.125, slopes=slopes, pos0=-1000)
    assert np.allclose(shifted, got, rtol=1e-11, atol=1e-13)


def test_alibi_with_zero_slopes_is_plain_attention_exactly():
    q, k, mask = _variant_inputs(64)
    got = oracle.attention_variants(q, k, mask=mask, scale=0.125, slopes=np.zeros(4))
    assert np.array_equal(got, oracle.attention(q, k, mask=mask, scale=0.125))


def test_sinks_match_brute_force():
    q, k, mask = _variant_inputs(65)
    sinks = np.array([-1.0, 0.0, 2.0, 7.5])
    got = oracle.attention_variants(q, k, mask=mask, scale=0.125, sinks=sinks)
    want = brute_force_variants(q, k, mask, 0.125, sinks=sinks)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12)


def test_a_minus_inf_sink_is_plain_attention_exactly():
    q, k, mask = _variant_inputs(66)
    got = oracle.attention_variants(q, k, mask=mask, scale=0.125, sinks=np.full(4, -np.inf))
    assert np.array_equal(got, oracle.attention(q, k, mask=mask, scale=0.125))


def test_sink_with_one_key_is_a_sigmoid():
    # one key of score s and a sink sigma: o = v * e^s / (e^s + e^sigma) = v * sigmoid(s - sigma)
    q, k, _ = _variant_inputs(67, n_q=1, H=3, n=1, masked=False)
    sinks = np.array([-0.5, 0.3, 4.0])
    got = oracle.attention_variants(q, k, scale=0.2, sinks=sinks)
    s = 0.2 * (q[0].astype(np.float64) @ k[0].astype(np.float64))
    want = k[0, :DV].astype(np.float64)[None, :] / (1.0 + np.exp(sinks - s))[:, None]
    assert np.allclose(got, want, rtol=1e-12, atol=1e-14)


def test_sink_on_a_fully_masked_row_gives_zero():
    q, k, mask = _variant_inputs(68, n_q=1)
    mask[:] = NEG
    got = oracle.attention_variants(q, k, mask=mask, scale=0.125, sinks=np.array([0.0, 1.0, 2.0, 3.0]))
    assert np.array_equal(got, np.zeros_like(got))


def test_all_variants_together_match_brute_force():
    q, k, mask = _variant_inputs(69, n_q=3, H=5, n=50)
    slopes = np.array([0.5, 0.25, 0.125, 0.0625, 0.03125])
    sinks = np.array([0.0, -2.0, 1.0, 3.0, -0.5])
    got = oracle.attention_variants(q, k, mask=mask, scale=0.1, softcap=3.0, slopes=slopes, pos0=47,
                                    sinks=sinks)
    want = brute_force_variants(q, k, mask, 0.1, softcap=3.0, slopes=slopes, pos0=47, sinks=sinks)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12)


# ---- log-sum-exp of a row and the merge of partial results (split-KV across devices) --

def test_lse_of_equal_scores_is_log_count():
    # Q = 0 and a zero mask: every score is 0, so lse = log(n) exactly
    rng = np.random.default_rng(40)
    for n in (1, 2, 7, 300):
        q = np.zeros((1, 3, DK), np.float16)
        k = rand_f16(rng, (n, DK))
        _, lse = oracle.attention_lse(q, k, mask=np.zeros((1, n), np.float16), scale=0.3)
        np.testing.assert_allclose(lse, np.full(3, math.log(n)), rtol=0, atol=1e-13)


def test_lse_with_a_one_hot_query_is_a_library_logsumexp():
    # q = e_c: the score of key j is scale * k[j, c] + mask[j], so the row's lse is
    # scipy's logsumexp of those numbers
    from scipy.special import logsumexp

    rng = np.random.default_rng(41)
    n, c, scale = 200, 517, 0.37
    k = rand_f16(rng, (n, DK), std=3.0)
    mask = rand_f16(rng, (1, n))
    mask[0, rng.random(n) < 0.3] = NEG
    q = np.zeros((1, 1, DK), np.float16)
    q[0, 0, c] = 1.0
    _, lse = oracle.attention_lse(q, k, mask=mask, scale=scale)
    s = scale * k[:, c].astype(np.float64) + mask[0].astype(np.float64)
    np.testing.assert_allclose(lse[0], logsumexp(s), rtol=0, atol=1e-12)


def test_lse_of_a_fully_masked_row_is_minus_inf_and_shifts_with_the_mask():
    rng = np.random.default_rng(42)
    q = rand_f16(rng, (2, 2, DK))
    k = rand_f16(rng, (50, DK))
    mask = np.zeros((2, 50), np.float16)
    mask[1, :] = NEG
    mask[0, 40:] = NEG
    _, lse = oracle.attention_lse(q, k, mask=mask, scale=0.07)
    assert np.all(np.isneginf(lse[2:])) and np.all(np.isfinite(lse[:2]))
    shifted = np.where(np.isneginf(mask), mask, mask + np.float16(6.0)).astype(np.float16)
    _, lse2 = oracle.attention_lse(q, k, mask=shifted, scale=0.07)
    np.testing.assert_allclose(lse2[:2], lse[:2] + 6.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("cuts", [(0, 300), (0, 100, 300), (0, 1, 150, 151, 300), (0, 60, 120, 300)])
def test_combine_of_key_range_parts_equals_the_whole(cuts):
    # attention over disjoint key ranges, merged by the log-sum-exp rule, is the
    # attention over all keys: pins the merge against the softmax definition. The
    # (0, 60, 120, 300) cut has a part whose keys are all masked (lse -inf).
    rng = np.random.default_rng(43)
    n = 300
    q = rand_f16(rng, (3, 4, DK))
    k = rand_f16(rng, (n, DK))
    mask = rand_f16(rng, (3, n))
    mask[:, 60:120] = NEG
    o_all, lse_all = oracle.attention_lse(q, k, mask=mask, scale=0.06)
    parts = [oracle.attention_lse(q, k[a:b], mask=mask[:, a:b], scale=0.06)
             for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = oracle.combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(o, o_all, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lse_all, rtol=0, atol=1e-12)


def test_combine_closed_forms():
    rng = np.random.default_rng(44)
    o = rng.standard_normal((2, 5, DV))
    lse0 = rng.standard_normal(5)
    # one part: the identity
    oo, ll = oracle.combine(o[:1], lse0[None])
    np.testing.assert_array_equal(oo, o[0])
    np.testing.assert_array_equal(ll, lse0)
    # weights 1 : 3
    lse = np.stack([lse0, lse0 + math.log(3.0)])
    oo, ll = oracle.combine(o, lse)
    np.testing.assert_allclose(oo, (o[0] + 3.0 * o[1]) / 4.0, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(ll, lse0 + math.log(4.0), rtol=0, atol=1e-13)
    # a -inf part is ignored; all parts -inf give 0 and -inf
    lse = np.stack([lse0, np.full(5, -np.inf)])
    oo, ll = oracle.combine(o, lse)
    np.testing.assert_array_equal(oo, o[0])
    oo, ll = oracle.combine(o, np.full((2, 5), -np.inf))
    assert np.all(oo == 0) and np.all(np.isneginf(ll))


# ---- the DK = DV = 512 head shape (V = the whole 512-wide row) ---------------------------

def test_dk512_matches_brute_force():
    rng = np.random.default_rng(50)
    q = rand_f16(rng, (3, 2, 512))
    k = rand_f16(rng, (37, 512))
    mask = rand_f16(rng, (3, 37))
    mask[1, ::3] = NEG
    got = oracle.attention(q, k, mask=mask, scale=0.05)
    np.testing.assert_allclose(got, brute_force(q, k, mask, 0.05), rtol=1e-12, atol=1e-13)


def test_dk512_single_key_gives_the_row():
    rng = np.random.default_rng(51)
    q = rand_f16(rng, (1, 4, 512))
    k = rand_f16(rng, (1, 512))
    got = oracle.attention(q, k, scale=0.3)
    np.testing.assert_array_equal(got, np.repeat(k.astype(np.float64), 4, axis=0))


def test_dk512_equals_dk576_with_zero_rope_columns_exactly():
    # 64 zero columns appended to q and to every cache row add exact zeros to each
    # score and leave V (the first 512 columns) as it is
    rng = np.random.default_rng(52)
    q = rand_f16(rng, (2, 3, 512))
    k = rand_f16(rng, (90, 512))
    mask = rand_f16(rng, (2, 90))
    mask[0, 40:] = NEG
    pad = lambda x: np.concatenate([x, np.zeros(x.shape[:-1] + (64,), np.float16)], axis=-1)
    o512, l512 = oracle.attention_lse(q, k, mask=mask, scale=0.07)
    o576, l576 = oracle.attention_lse(pad(q), pad(k), mask=mask, scale=0.07)
    np.testing.assert_array_equal(o512, o576)
    np.testing.assert_array_equal(l512, l576)


def test_planted_merge_and_lse_mistakes_are_caught():
    """Plausible mistakes in the merge and the lse, planted in numpy copies on the CPU:
    weights exp(lse) without the max shift (overflow), the lse in log2 units, the merge
    weighting by e^{-lse}, and the lse without the mask. Each must fail a pin above."""
    rng = np.random.default_rng(45)
    n = 120
    q = rand_f16(rng, (2, 3, DK))
    k = rand_f16(rng, (n, DK))
    mask = rand_f16(rng, (2, n))
    o_all, lse_all = oracle.attention_lse(q, k, mask=mask, scale=0.06)
    parts = [oracle.attention_lse(q, k[a:b], mask=mask[:, a:b], scale=0.06)
             for a, b in ((0, 50), (50, 120))]
    o_p = np.stack([p[0] for p in parts])
    l_p = np.stack([p[1] for p in parts])

    def merge(o, lse, w_of):
        w = w_of(lse)
        return (w[:, :, None] * o).sum(0) / w.sum(0)[:, None]

    # the real merge reproduces the whole
    good, _ = oracle.combine(o_p, l_p)
    np.testing.assert_allclose(good, o_all, rtol=1e-12, atol=1e-13)
    # weights by e^{-lse}: wrong result
    assert np.max(np.abs(merge(o_p, l_p, lambda l: np.exp(-l)) - o_all)) > 1e-3
    # no max shift: with large lse values the weights overflow to inf and the merge is NaN
    with np.errstate(over="ignore", invalid="ignore"):
        assert not np.all(np.isfinite(merge(o_p, l_p + 800.0, np.exp)))
    shifted, _ = oracle.combine(o_p, l_p + 800.0)  # the real merge is shift invariant
    np.testing.assert_allclose(shifted, good, rtol=1e-12, atol=1e-13)
    # lse in log2 units, or without the mask: the one-hot / log(n) pins disagree
    qz = np.zeros((1, 1, DK), np.float16)
    _, l_ok = oracle.attention_lse(qz, k[:7], mask=np.zeros((1, 7), np.float16), scale=0.3)
    assert abs(l_ok[0] - math.log(7)) < 1e-13
    assert abs(l_ok[0] / math.log(2) - math.log(7)) > 1e-3
    m1 = np.full((1, 7), np.float16(2.0))
    _, l_m = oracle.attention_lse(qz, k[:7], mask=m1, scale=0.3)
    assert abs(l_m[0] - (math.log(7) + 2.0)) < 1e-12 and abs(l_m[0] - math.log(7)) > 1.0


# ---- attention with a K and a V per KV head (the DK = 192 / DV = 128 head shape) --------

def _loop_heads(q, k, v, mask, scale):
    """The same definition by explicit per-row loops (no einsum, no grouping trick)."""
    n_q, H, _ = q.shape
    n, Hkv, _ = k.shape
    out = np.zeros((n_q * H, v.shape[2]))
    for t in range(n_q):
        for h in range(H):
            hk = h // (H // Hkv)
            s = [scale * float(np.dot(q[t, h].astype(np.float64), k[j, hk].astype(np.float64)))
                 + (0.0 if mask is None else float(mask[t, j])) for j in range(n)]
            mx = max(s)
            if mx == -math.inf:
                continue
            w = [math.exp(x - mx) for x in s]
            tot = math.fsum(w)
            out[t * H + h] = sum(wj * v[j, hk].astype(np.float64) for j, wj in enumerate(w)) / tot
    return out


@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (6, 1)])
def test_heads_match_explicit_loops(H, Hkv):
    rng = np.random.default_rng(70 + H + Hkv)
    q = rand_f16(rng, (3, H, 192))
    k = rand_f16(rng, (11, Hkv, 192))
    v = rand_f16(rng, (11, Hkv, 128))
    mask = rand_f16(rng, (3, 11))
    mask[2, :] = NEG  # a token with nothing kept
    mask[0, 4] = NEG
    got = oracle.attention_heads(q, k, v, mask, 0.08)
    np.testing.assert_allclose(got, _loop_heads(q, k, v, mask, 0.08), rtol=1e-12, atol=1e-13)
    assert np.all(got[2 * H:] == 0)


def test_heads_single_key_gives_its_value_row():
    rng = np.random.default_rng(71)
    q = rand_f16(rng, (2, 4, 192))
    k = rand_f16(rng, (1, 2, 192))
    v = rand_f16(rng, (1, 2, 128))
    got = oracle.attention_heads(q, k, v, None, 0.3).reshape(2, 4, 128)
    for h in range(4):
        np.testing.assert_array_equal(got[:, h], np.broadcast_to(v[0, h // 2].astype(np.float64), (2, 128)))


def test_heads_with_one_shared_head_is_the_mla_attention():
    # one KV head, dk = 576 and V = the first 512 columns of K: the C oracle's MLA
    # attention, an independent implementation of the same definition
    rng = np.random.default_rng(72)
    q = rand_f16(rng, (2, 5, DK))
    kc = rand_f16(rng, (60, DK))
    mask = rand_f16(rng, (2, 60))
    mask[1, 10:20] = NEG
    got = oracle.attention_heads(q, kc[:, None, :], kc[:, None, :DV], mask, 0.05)
    np.testing.assert_allclose(got, oracle.attention(q, kc, mask=mask, scale=0.05), rtol=1e-11, atol=1e-12)


def test_heads_permuting_kv_heads_with_their_groups_permutes_the_output():
    rng = np.random.default_rng(73)
    H, Hkv = 6, 3
    q = rand_f16(rng, (2, H, 192))
    k = rand_f16(rng, (20, Hkv, 192))
    v = rand_f16(rng, (20, Hkv, 128))
    base = oracle.attention_heads(q, k, v, None, 0.07).reshape(2, H, 128)
    perm = np.array([2, 0, 1])
    qperm = np.concatenate([q[:, 2 * p:2 * p + 2] for p in perm], axis=1)
    got = oracle.attention_heads(qperm, k[:, perm], v[:, perm], None, 0.07).reshape(2, H, 128)
    want = np.concatenate([base[:, 2 * p:2 * p + 2] for p in perm], axis=1)
    np.testing.assert_array_equal(got, want)
