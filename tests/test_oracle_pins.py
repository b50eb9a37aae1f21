"""Pins of the fp64 CPU oracle to facts outside itself (CPU only).

Each check targets a part of the oracle with a value fixed by the mathematics or the pages, so that a
plausible slip (a dropped scale, a wrong sign, a transposed operand, an off-by-one causal mask, a
wrong LSE base, a bad group merge) fails at least one of them:

  * hand-derived worked examples (tests/golden/hand_examples.json);
  * Q = 0 closed form: O is the mean of the visible V rows, LSE = ln(#visible keys);
  * causal row 0: O_0 = V_0, LSE_0 = scale * q_0 . k_0;
  * a library softmax / logsumexp (scipy) applied to the same scores;
  * key-shift invariance: K + 1 c^T leaves O unchanged and shifts LSE by scale * q . c;
  * joint permutation of K and V rows leaves non-causal results unchanged (position independence
    of exact attention, "Was FlashAttention bei Transformer-Inference verändert");
  * linearity in V;
  * scalar brute force (math.fsum) on tiny inputs, all mask kinds;
  * the tiled online-softmax loop and the 3-group merge of "轻松读懂FlashAttention 上" against the
    materialised definition;
  * padded + 2-D key mask against packed varlen (to rounding, on valid rows);
  * split-KV partials + combine against the materialised single-query result;
  * safe softmax: huge scores stay finite ("小知识" note under "内存卡点");
  * the prefix-LM mask: the Q = 0 closed form with its visible-key count, the limits prefix = 0
    (causal) and prefix >= Nk (no mask), invariance under permutations inside the prefix (the prefix
    is bidirectional), brute force, the row sampler and the packed varlen form;
  * decode with grouped KV heads and per-sequence cache lengths: equal to the dense decode over KV
    heads repeated G times, equal to decode over the truncated cache, the Q = 0 closed form, and
    the split-KV combine with empty splits;
  * decode over key shards of a cache: the Q = 0 closed form with the shard's own visible-key
    count, and the merge of all shards' results equal to decode over the whole cache;
  * the backward (dQ, dK, dV): central finite differences of the forward oracle (causal, unmasked,
    prefix-LM, and the packed varlen form), the Q = 0 closed forms, invariance of dQ and dV under a
    common key shift, and zero total dK; the row-sampled backward for long heads equals the
    whole-head backward at every row and column.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle
import seeded_inputs as si

RTOL = 1e-12


def rnd(shape, seed, dtype="bf16"):
    bits = si.normal_bits([99, seed], int(np.prod(shape)), dtype)
    return si.bits_to_float(bits, dtype).reshape(shape)


# ---------------------------------------------------------------------------------------------
# hand-derived golden cases


def _f(x):
    return -math.inf if x == "-inf" else float(x)


def _golden_cases(golden_dir):
    with open(os.path.join(golden_dir, "hand_examples.json")) as fh:
        return json.load(fh)["cases"]


def test_hand_examples_materialised(golden_dir):
    for c in _golden_cases(golden_dir):
        o, lse = oracle.attention_head(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]),
                                       c["scale"], c["causal"])
        np.testing.assert_allclose(o, np.array(c["o"]), rtol=0, atol=1e-13, err_msg=c["name"])
        exp_lse = np.array([_f(x) for x in c["lse"]])
        assert np.array_equal(np.isinf(lse), np.isinf(exp_lse)), c["name"]
        fin = np.isfinite(exp_lse)
        np.testing.assert_allclose(lse[fin], exp_lse[fin], rtol=0, atol=1e-13, err_msg=c["name"])


def test_hand_examples_brute_and_tiled(golden_dir):
    for c in _golden_cases(golden_dir):
        exp_o = np.array(c["o"])
        exp_lse = np.array([_f(x) for x in c["lse"]])
        bo, bl = oracle.brute_attention_head(c["q"], c["k"], c["v"], c["scale"], c["causal"])
        to, tl = oracle.tiled_online_attention(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]),
                                               c["scale"], c["causal"], block_q=2, block_k=2)
        for o, lse in ((np.array(bo), np.array(bl)), (to, tl)):
            np.testing.assert_allclose(o, exp_o, rtol=0, atol=1e-13, err_msg=c["name"])
            fin = np.isfinite(exp_lse)
            assert np.array_equal(np.isfinite(lse), fin), c["name"]
            np.testing.assert_allclose(lse[fin], exp_lse[fin], rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------------------------
# closed forms


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_closed_form(causal):
    n, d = 37, 8
    q = np.zeros((n, d))
    k = rnd((n, d), 1)
    v = rnd((n, d), 2)
    o, lse = oracle.attention_head(q, k, v, scale=0.3, causal=causal)
    for i in range(n):
        vis = i + 1 if causal else n
        np.testing.assert_allclose(o[i], v[:vis].mean(axis=0), rtol=RTOL, atol=1e-14)
        assert abs(lse[i] - math.log(vis)) < 1e-13


def test_causal_row_zero_closed_form():
    n, d = 20, 16
    q, k, v = rnd((n, d), 3), rnd((n, d), 4), rnd((n, d), 5)
    scale = 0.125
    o, lse = oracle.attention_head(q, k, v, scale, causal=True)
    np.testing.assert_array_equal(o[0], v[0])
    assert abs(lse[0] - scale * float(np.dot(q[0], k[0]))) < 1e-13


def test_single_key_returns_value_row():
    q, k, v = rnd((5, 4), 6), rnd((1, 4), 7), rnd((1, 3), 8)
    o, lse = oracle.attention_head(q, k, v, 0.7)
    np.testing.assert_array_equal(o, np.repeat(v, 5, axis=0))
    np.testing.assert_allclose(lse, 0.7 * (q @ k[0]), rtol=1e-15)


# ---------------------------------------------------------------------------------------------
# library routines


@pytest.mark.parametrize("scale", [0.125, 1.0 / math.sqrt(128), 0.1])
def test_matches_scipy_softmax_noncausal(scale):
    nq, nk, d, dv = 19, 23, 16, 12
    q, k, v = rnd((nq, d), 9), rnd((nk, d), 10), rnd((nk, dv), 11)
    o, lse = oracle.attention_head(q, k, v, scale)
    scores = scale * np.einsum("id,jd->ij", q, k)
    np.testing.assert_allclose(o, scipy.special.softmax(scores, axis=1) @ v, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(scores, axis=1), rtol=1e-13)


def test_matches_scipy_softmax_causal_rectangular():
    nq, nk, d = 7, 12, 8
    q, k, v = rnd((nq, d), 12), rnd((nk, d), 13), rnd((nk, d), 14)
    o, lse = oracle.attention_head(q, k, v, 0.4, causal=True)
    for i in range(nq):
        last = i + (nk - nq) + 1
        sc = 0.4 * np.array([np.dot(q[i], k[j]) for j in range(last)])
        np.testing.assert_allclose(o[i], scipy.special.softmax(sc) @ v[:last], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[i], scipy.special.logsumexp(sc), rtol=1e-13)


# ---------------------------------------------------------------------------------------------
# invariants


def test_key_shift_invariance():
    nq, nk, d = 9, 15, 8
    q, k, v = rnd((nq, d), 15), rnd((nk, d), 16), rnd((nk, d), 17)
    c = rnd((d,), 18)
    scale = 0.37
    o1, l1 = oracle.attention_head(q, k, v, scale)
    o2, l2 = oracle.attention_head(q, k + c[None, :], v, scale)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(l2, l1 + scale * (q @ c), rtol=1e-12, atol=1e-12)


def test_joint_key_value_permutation_invariance():
    nq, nk, d = 11, 29, 8
    q, k, v = rnd((nq, d), 19), rnd((nk, d), 20), rnd((nk, d), 21)
    perm = np.random.default_rng(0).permutation(nk)
    o1, l1 = oracle.attention_head(q, k, v, 0.2)
    o2, l2 = oracle.attention_head(q, k[perm], v[perm], 0.2)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l2, l1, rtol=1e-13)


def test_linear_in_values():
    nq, nk, d = 6, 10, 4
    q, k = rnd((nq, d), 22), rnd((nk, d), 23)
    v1, v2 = rnd((nk, 5), 24), rnd((nk, 5), 25)
    a = rnd((5, 3), 26)
    o1, _ = oracle.attention_head(q, k, v1, 0.5, causal=True)
    o2, _ = oracle.attention_head(q, k, v2, 0.5, causal=True)
    o12, _ = oracle.attention_head(q, k, v1 + v2, 0.5, causal=True)
    oa, _ = oracle.attention_head(q, k, v1 @ a, 0.5, causal=True)
    np.testing.assert_allclose(o12, o1 + o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(oa, o1 @ a, rtol=1e-12, atol=1e-13)


def test_safe_softmax_stays_finite():
    q = np.array([[1.0, 0.0], [0.0, 1.0]])
    k = np.array([[3000.0, 0.0], [2990.0, 1.0], [0.0, 5000.0]])
    v = np.array([[1.0], [2.0], [3.0]])
    o, lse = oracle.attention_head(q, k, v, 1.0)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    # row 0: scores 3000, 2990, 0 -> weights ~ (1, e^-10, 0)
    w = np.array([1.0, math.exp(-10.0)])
    np.testing.assert_allclose(o[0, 0], (w @ [1.0, 2.0]) / w.sum(), rtol=1e-14)
    np.testing.assert_allclose(lse[0], 3000.0 + math.log(w.sum()), rtol=1e-15)


# ---------------------------------------------------------------------------------------------
# brute force on tiny inputs


@pytest.mark.parametrize("nq,nk,causal,k_valid", [
    (1, 1, False, None), (4, 4, True, None), (5, 9, True, None), (9, 5, True, None),
    (16, 16, False, 11), (7, 13, False, None), (16, 16, True, None), (3, 16, False, 1),
])
def test_matches_brute_force(nq, nk, causal, k_valid):
    d, dv = 6, 5
    q, k, v = rnd((nq, d), 30 + nq), rnd((nk, d), 40 + nk), rnd((nk, dv), 50 + nk)
    o, lse = oracle.attention_head(q, k, v, 0.3, causal, k_valid)
    bo, bl = oracle.brute_attention_head(q.tolist(), k.tolist(), v.tolist(), 0.3, causal, k_valid)
    bo, bl = np.array(bo), np.array(bl)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-14)
    assert np.array_equal(np.isfinite(lse), np.isfinite(bl))
    fin = np.isfinite(bl)
    np.testing.assert_allclose(lse[fin], bl[fin], rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------------------------------------
# the tiled algorithm and the group merge against the definition


@pytest.mark.parametrize("nq,nk,causal,bq,bk,k_valid", [
    (300, 300, True, 128, 128, None), (300, 300, False, 128, 128, None),
    (257, 513, True, 64, 128, None), (129, 77, True, 32, 16, None),
    (200, 200, False, 128, 128, 133), (64, 64, True, 64, 64, None),
])
def test_tiled_online_matches_materialised(nq, nk, causal, bq, bk, k_valid):
    d = 16
    q, k, v = rnd((nq, d), 60), rnd((nk, d), 61), rnd((nk, d), 62)
    o, lse = oracle.attention_head(q, k, v, 0.25, causal, k_valid)
    to, tl = oracle.tiled_online_attention(q, k, v, 0.25, causal, bq, bk, k_valid)
    np.testing.assert_allclose(to, o, rtol=1e-12, atol=1e-13)
    fin = np.isfinite(lse)
    assert np.array_equal(np.isfinite(tl), fin)
    np.testing.assert_allclose(tl[fin], lse[fin], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("n,groups", [(3, 3), (10, 3), (100, 3), (1000, 7), (5, 5)])
def test_group_merge_equals_full_softmax(n, groups):
    x = 3.0 * rnd((n,), 70 + n)
    p, m, l = oracle.softmax_by_groups(x, groups)
    np.testing.assert_allclose(p, scipy.special.softmax(x), rtol=1e-12, atol=1e-300)
    assert m == x.max()
    np.testing.assert_allclose(m + math.log(l), scipy.special.logsumexp(x), rtol=1e-14)


def test_group_merge_order_independent_of_max_position():
    x = np.array([0.0, 1.0, 50.0, -3.0, 2.0, 49.5])
    p_a, _, _ = oracle.softmax_by_groups(x, 3)
    p_b, _, _ = oracle.softmax_by_groups(x, 2)
    p_c, _, _ = oracle.softmax_by_groups(x, 6)
    np.testing.assert_allclose(p_a, p_b, rtol=1e-14)
    np.testing.assert_allclose(p_a, p_c, rtol=1e-14)


# ---------------------------------------------------------------------------------------------
# varlen / key padding


def test_padded_key_mask_equals_packed_varlen():
    lengths = [5, 17, 1, 12]
    H, D = 2, 8
    q, k, v, cu = si.varlen_qkv(7, lengths, H, D, "fp16")
    qf, kf, vf = (si.bits_to_float(t, "fp16") for t in (q, k, v))
    o_p, l_p = oracle.attention_varlen(qf, kf, vf, cu, 0.1)
    nmax = max(lengths)
    B = len(lengths)
    pad = lambda t: np.stack([np.pad(t[cu[b]:cu[b + 1]], ((0, nmax - lengths[b]), (0, 0), (0, 0)),
                                     constant_values=7.0) for b in range(B)])
    mask = np.array([[j < lengths[b] for j in range(nmax)] for b in range(B)])
    o_d, l_d = oracle.padded_key_mask_attention(pad(qf), pad(kf), pad(vf), mask, 0.1)
    for b in range(B):
        L = lengths[b]
        # equal up to the summation order of the BLAS products (padded rows change the blocking)
        np.testing.assert_allclose(o_d[b, :L], o_p[cu[b]:cu[b + 1]], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(l_d[b, :, :L], l_p[:, cu[b]:cu[b + 1]], rtol=1e-14, atol=1e-14)


def test_varlen_key_valid_equals_truncation():
    n, d = 40, 8
    q, k, v = rnd((n, d), 80), rnd((n, d), 81), rnd((n, d), 82)
    o1, l1 = oracle.attention_head(q, k, v, 0.3, k_valid=23)
    o2, l2 = oracle.attention_head(q, k[:23], v[:23], 0.3)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-14)


# ---------------------------------------------------------------------------------------------
# decode: split-KV partials + combine


@pytest.mark.parametrize("nk,splits", [(64, 1), (64, 16), (100, 16), (37, 3), (5, 16), (8192, 16)])
def test_split_kv_combine_equals_full(nk, splits):
    d = 32
    q, k, v = rnd((d,), 90), rnd((nk, d), 91), rnd((nk, d), 92)
    scale = 1.0 / math.sqrt(d)
    o_ref, l_ref = oracle.attention_head(q[None, :], k, v, scale)
    parts_o, parts_l = oracle.split_kv_partials(q, k, v, scale, splits)
    o, lse = oracle.combine_partials(parts_o, parts_l)
    np.testing.assert_allclose(o, o_ref[0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, l_ref[0], rtol=1e-13)
    # each partial is itself the attention over its own key range
    for s, (lo, hi) in enumerate(oracle.online.split_bounds(nk, splits)):
        if hi > lo:
            po, pl = oracle.attention_head(q[None, :], k[lo:hi], v[lo:hi], scale)
            np.testing.assert_allclose(parts_o[s], po[0], rtol=1e-12, atol=1e-14)
        else:
            assert parts_l[s] == -np.inf


def test_row_sampler_matches_full_head():
    nq, nk, d = 70, 70, 8
    q, k, v = rnd((nq, d), 93), rnd((nk, d), 94), rnd((nk, d), 95)
    rows = [0, 1, 33, 69]
    for causal in (False, True):
        o, lse = oracle.attention_head(q, k, v, 0.5, causal)
        ro, rl = oracle.attention_rows(q, k, v, rows, 0.5, causal)
        np.testing.assert_allclose(ro, o[rows], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(rl, lse[rows], rtol=1e-13)


# ---------------------------------------------------------------------------------------------
# prefix-LM mask (causal with a bidirectional prefix of keys)


@pytest.mark.parametrize("nq,nk,prefix", [(37, 37, 5), (20, 33, 9), (33, 20, 4), (16, 16, 40)])
def test_prefix_zero_query_closed_form(nq, nk, prefix):
    # Q = 0: every visible key has the same score, so O_i is the mean of the visible V rows and
    # LSE_i = ln(#visible) with #visible = min(Nk, max(prefix, i + 1 + Nk - Nq)) (0 -> O = 0, -inf)
    d = 8
    q = np.zeros((nq, d))
    k, v = rnd((nk, d), 101), rnd((nk, d), 102)
    o, lse = oracle.attention_head(q, k, v, scale=0.3, causal=True, prefix=prefix)
    for i in range(nq):
        vis = min(nk, max(prefix, i + 1 + nk - nq))
        if vis <= 0:
            assert np.all(o[i] == 0) and lse[i] == -math.inf
            continue
        np.testing.assert_allclose(o[i], v[:vis].mean(axis=0), rtol=RTOL, atol=1e-14)
        assert abs(lse[i] - math.log(vis)) < 1e-13


def test_prefix_limits_are_causal_and_full():
    nq, nk, d = 23, 23, 8
    q, k, v = rnd((nq, d), 103), rnd((nk, d), 104), rnd((nk, d), 105)
    oc, lc = oracle.attention_head(q, k, v, 0.25, causal=True)
    o0, l0 = oracle.attention_head(q, k, v, 0.25, causal=True, prefix=0)
    np.testing.assert_array_equal(o0, oc)
    np.testing.assert_array_equal(l0, lc)
    of, lf = oracle.attention_head(q, k, v, 0.25, causal=False)
    on, ln = oracle.attention_head(q, k, v, 0.25, causal=True, prefix=nk)
    np.testing.assert_array_equal(on, of)
    np.testing.assert_array_equal(ln, lf)


def test_prefix_keys_are_bidirectional():
    # permuting keys (jointly with their values) inside the prefix leaves every row unchanged, which
    # a causal treatment of the prefix would not
    nq, nk, d, prefix = 19, 19, 8, 7
    q, k, v = rnd((nq, d), 106), rnd((nk, d), 107), rnd((nk, d), 108)
    perm = np.concatenate([np.random.default_rng(1).permutation(prefix), np.arange(prefix, nk)])
    o1, l1 = oracle.attention_head(q, k, v, 0.2, causal=True, prefix=prefix)
    o2, l2 = oracle.attention_head(q, k[perm], v[perm], 0.2, causal=True, prefix=prefix)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l2, l1, rtol=1e-13)
    oc, _ = oracle.attention_head(q, k, v, 0.2, causal=True)
    assert not np.allclose(o1[:prefix], oc[:prefix])  # the prefix rows do see later prefix keys


@pytest.mark.parametrize("nq,nk,prefix", [(6, 6, 3), (5, 9, 2), (9, 5, 4), (16, 16, 1), (7, 13, 13)])
def test_prefix_matches_brute_force(nq, nk, prefix):
    d, dv = 6, 5
    q, k, v = rnd((nq, d), 110 + nq), rnd((nk, d), 120 + nk), rnd((nk, dv), 130 + nk)
    o, lse = oracle.attention_head(q, k, v, 0.3, True, prefix=prefix)
    bo, bl = oracle.brute_attention_head(q.tolist(), k.tolist(), v.tolist(), 0.3, True, prefix=prefix)
    bo, bl = np.array(bo), np.array(bl)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-14)
    assert np.array_equal(np.isfinite(lse), np.isfinite(bl))
    fin = np.isfinite(bl)
    np.testing.assert_allclose(lse[fin], bl[fin], rtol=1e-13, atol=1e-14)


def test_prefix_row_sampler_and_varlen():
    nq, d, prefix = 70, 8, 25
    q, k, v = rnd((nq, d), 131), rnd((nq, d), 132), rnd((nq, d), 133)
    o, lse = oracle.attention_head(q, k, v, 0.5, True, prefix=prefix)
    rows = [0, 1, 24, 25, 26, 69]
    ro, rl = oracle.attention_rows(q, k, v, rows, 0.5, True, prefix=prefix)
    np.testing.assert_allclose(ro, o[rows], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(rl, lse[rows], rtol=1e-13)
    # packed varlen: the prefix counts from each sequence's first key
    cu = [0, 30, 70]
    qp, kp, vp = q[:, None, :], k[:, None, :], v[:, None, :]
    vo, vl = oracle.attention_varlen(qp, kp, vp, cu, 0.5, causal=True, prefix=prefix)
    for b in range(2):
        s0, s1 = cu[b], cu[b + 1]
        eo, el = oracle.attention_head(q[s0:s1], k[s0:s1], v[s0:s1], 0.5, True, prefix=prefix)
        np.testing.assert_array_equal(vo[s0:s1, 0], eo)
        np.testing.assert_array_equal(vl[0, s0:s1], el)


# ---------------------------------------------------------------------------------------------
# decode with grouped KV heads and per-sequence cache lengths


def test_gqa_decode_equals_replicated_kv_heads():
    # grouped heads are the dense decode over K/V heads repeated G times along the head axis
    B, Nk, Hkv, G, D = 3, 50, 2, 4, 8
    q = rnd((B, 1, Hkv * G, D), 140)
    k, v = rnd((B, Nk, Hkv, D), 141), rnd((B, Nk, Hkv, D), 142)
    o, lse = oracle.attention_decode_gqa(q, k, v, 0.3)
    o_ref, lse_ref = oracle.attention_decode(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), 0.3)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, lse_ref[:, :, 0])


def test_gqa_decode_lengths_truncate_the_cache():
    B, Nk, Hkv, G, D = 4, 40, 3, 2, 8
    q = rnd((B, 1, Hkv * G, D), 143)
    k, v = rnd((B, Nk, Hkv, D), 144), rnd((B, Nk, Hkv, D), 145)
    lens = [40, 1, 17, 0]
    o, lse = oracle.attention_decode_gqa(q, k, v, 0.25, lens)
    for b, L in enumerate(lens):
        if L == 0:
            assert np.all(o[b] == 0) and np.all(lse[b] == -np.inf)
            continue
        ob, lb = oracle.attention_decode_gqa(q[b:b + 1], k[b:b + 1, :L], v[b:b + 1, :L], 0.25)
        np.testing.assert_array_equal(o[b], ob[0])
        np.testing.assert_array_equal(lse[b], lb[0])


def test_gqa_decode_zero_query_closed_form():
    # Q = 0: O is the mean of the first L value rows of the KV head, LSE = ln L
    B, Nk, Hkv, G, D = 2, 30, 2, 3, 8
    q = np.zeros((B, 1, Hkv * G, D))
    k, v = rnd((B, Nk, Hkv, D), 146), rnd((B, Nk, Hkv, D), 147)
    lens = [30, 7]
    o, lse = oracle.attention_decode_gqa(q, k, v, 0.5, lens)
    for b, L in enumerate(lens):
        for h in range(Hkv * G):
            np.testing.assert_allclose(o[b, 0, h], v[b, :L, h // G].mean(axis=0), rtol=RTOL, atol=1e-14)
            assert abs(lse[b, h] - math.log(L)) < 1e-13


def test_combine_of_empty_splits():
    # splits past a short cache carry LSE = -inf and contribute nothing; the combine equals the
    # materialised result
    nk, splits, d = 5, 16, 8
    q, k, v = rnd((d,), 148), rnd((nk, d), 149), rnd((nk, d), 150)
    parts = oracle.split_kv_partials(q, k, v, 0.4, splits)
    o, lse = oracle.combine_partials(*parts)
    o_ref, lse_ref = oracle.attention_head(q[None, :], k, v, 0.4)
    np.testing.assert_allclose(o, o_ref[0], rtol=1e-12, atol=1e-14)
    assert abs(lse - lse_ref[0]) < 1e-12


def test_shard_results_merge_to_the_whole_cache():
    # decode over contiguous key shards, merged with the split-KV combine, equals decode over the
    # whole cache, for lengths ending inside, at the edge of, and before a shard (and 0)
    B, Nk, Hkv, G, D = 5, 50, 2, 2, 8
    q = rnd((B, 1, Hkv * G, D), 151)
    k, v = rnd((B, Nk, Hkv, D), 152), rnd((B, Nk, Hkv, D), 153)
    lens = [50, 17, 0, 35, 20]
    bounds = [(0, 20), (20, 35), (35, 50)]
    shards = [oracle.attention_decode_shard(q, k[:, lo:hi], v[:, lo:hi], 0.35, lo, lens) for lo, hi in bounds]
    o_ref, lse_ref = oracle.attention_decode_gqa(q, k, v, 0.35, lens)
    for b in range(B):
        for h in range(Hkv * G):
            o, lse = oracle.combine_partials([s[0][b, 0, h] for s in shards], [s[1][b, h] for s in shards])
            if lens[b] == 0:
                assert np.all(o == 0) and lse == -np.inf and lse_ref[b, h] == -np.inf
                continue
            np.testing.assert_allclose(o, o_ref[b, 0, h], rtol=1e-12, atol=1e-14)
            assert abs(lse - lse_ref[b, h]) < 1e-12


def test_shard_decode_zero_query_closed_form():
    # Q = 0: a shard's O is the mean of ITS visible value rows and its LSE is ln(#visible keys of the
    # shard), here keys [20, 30) of the whole cache with whole-cache lengths 25, 20, 40, 30
    B, Nk_shard, Hkv, D, off = 4, 10, 1, 8, 20
    q = np.zeros((B, 1, 2, D))
    k, v = rnd((B, Nk_shard, Hkv, D), 154), rnd((B, Nk_shard, Hkv, D), 155)
    o, lse = oracle.attention_decode_shard(q, k, v, 0.5, off, [25, 20, 40, 30])
    for b, n in enumerate([5, 0, 10, 10]):
        for h in range(2):
            if n == 0:
                assert np.all(o[b, 0, h] == 0) and lse[b, h] == -np.inf
                continue
            np.testing.assert_allclose(o[b, 0, h], v[b, :n, 0].mean(axis=0), rtol=RTOL, atol=1e-14)
            assert abs(lse[b, h] - math.log(n)) < 1e-13


# ---------------------------------------------------------------------------------------------
# decode over a paged cache (page pool + per-sequence block table)


def _paginate(k, v, ps, rng):
    """Cut a contiguous cache [B, Nk, Hkv, D] into pages of ps rows, laid into a shuffled pool with a
    few spare pages; returns the pool, the block table and the spare page indices."""
    B, Nk = k.shape[:2]
    npg = -(-Nk // ps)
    pool_n = B * npg + 3
    perm = rng.permutation(pool_n)
    kp = np.full((pool_n, ps) + k.shape[2:], 7.0)
    vp = np.full((pool_n, ps) + v.shape[2:], 7.0)
    table = np.zeros((B, npg), dtype=np.int64)
    for b in range(B):
        for i in range(npg):
            page = int(perm[b * npg + i])
            table[b, i] = page
            rows = slice(i * ps, min((i + 1) * ps, Nk))
            kp[page, :rows.stop - rows.start] = k[b, rows]
            vp[page, :rows.stop - rows.start] = v[b, rows]
    return kp, vp, table, [int(x) for x in perm[B * npg:]]


def test_paged_decode_equals_contiguous_decode():
    # the same keys in shuffled pages through a table give the contiguous result, bit for bit, for
    # lengths ending inside a page, at a page edge, at one key, and at zero
    B, Nk, Hkv, G, D, ps = 5, 37, 2, 3, 8, 8
    rng = np.random.default_rng(160)
    q = rnd((B, 1, Hkv * G, D), 161)
    k, v = rnd((B, Nk, Hkv, D), 162), rnd((B, Nk, Hkv, D), 163)
    lens = [37, 16, 1, 0, 9]
    kp, vp, table, _ = _paginate(k, v, ps, rng)
    o, lse = oracle.attention_decode_paged(q, kp, vp, table, 0.3, lens)
    o_ref, lse_ref = oracle.attention_decode_gqa(q, k, v, 0.3, lens)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, lse_ref)


def test_paged_decode_reads_only_the_named_pages():
    # table entries past ceil(L / page_size) and pages no entry names may hold anything (here NaN
    # pages and entry -1): the result is unchanged
    B, Nk, Hkv, G, D, ps = 3, 24, 1, 2, 8, 4
    rng = np.random.default_rng(164)
    q = rnd((B, 1, Hkv * G, D), 165)
    k, v = rnd((B, Nk, Hkv, D), 166), rnd((B, Nk, Hkv, D), 167)
    lens = [24, 10, 3]
    kp, vp, table, spare = _paginate(k, v, ps, rng)
    o_ref, lse_ref = oracle.attention_decode_paged(q, kp, vp, table, 0.4, lens)
    kp2, vp2, t2 = kp.copy(), vp.copy(), table.copy()
    for b, L in enumerate(lens):
        for i in range(-(-L // ps), t2.shape[1]):
            kp2[t2[b, i]] = np.nan
            vp2[t2[b, i]] = np.nan
            t2[b, i] = -1
    for page in spare:
        kp2[page] = np.nan
        vp2[page] = np.nan
    o, lse = oracle.attention_decode_paged(q, kp2, vp2, t2, 0.4, lens)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, lse_ref)


def test_paged_decode_zero_query_closed_form():
    # Q = 0: O is the mean of the first L value rows in table order, LSE = ln L
    B, Hkv, G, D, ps = 3, 2, 2, 8, 4
    rng = np.random.default_rng(168)
    pool = 9
    vp = rnd((pool, ps, Hkv, D), 169)
    kp = rnd((pool, ps, Hkv, D), 170)
    table = np.array([rng.permutation(pool)[:3] for _ in range(B)])
    lens = [12, 5, 1]
    q = np.zeros((B, 1, Hkv * G, D))
    o, lse = oracle.attention_decode_paged(q, kp, vp, table, 0.7, lens)
    for b, L in enumerate(lens):
        rows = np.concatenate([vp[p] for p in table[b]])[:L]
        for h in range(Hkv * G):
            np.testing.assert_allclose(o[b, 0, h], rows[:, h // G].mean(axis=0), rtol=RTOL, atol=1e-14)
            assert abs(lse[b, h] - math.log(L)) < 1e-13


def test_paged_decode_brute_force():
    # tiny case against scalar evaluation over the keys gathered row by row through the table
    Hkv, G, D, ps = 1, 2, 3, 2
    kp, vp = rnd((4, ps, Hkv, D), 171), rnd((4, ps, Hkv, D), 172)
    table = np.array([[2, 0, 3]])
    L = 5
    q = rnd((1, 1, Hkv * G, D), 173)
    o, lse = oracle.attention_decode_paged(q, kp, vp, table, 0.9, [L])
    keys = [kp[table[0, j // ps], j % ps, 0] for j in range(L)]
    vals = [vp[table[0, j // ps], j % ps, 0] for j in range(L)]
    for h in range(G):
        ob, lb = oracle.brute_attention_head(q[0, :, h], np.array(keys), np.array(vals), 0.9)
        np.testing.assert_allclose(o[0, 0, h], ob[0], rtol=1e-12, atol=1e-14)
        assert abs(lse[0, h] - lb[0]) < 1e-12


# ---------------------------------------------------------------------------------------------
# backward: the derivative of the forward definition


def _loss(q, k, v, do, scale, causal, prefix=0):
    o, _ = oracle.attention_head(q, k, v, scale, causal, prefix=prefix)
    return float((o * do).sum())


def _central_differences(loss, tensors, h=1e-5):
    """d loss / d x for every element of every tensor (edited in place and restored)."""
    out = []
    for x in tensors:
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + h
            lp = loss()
            x[idx] = keep - h
            lm = loss()
            x[idx] = keep
            num[idx] = (lp - lm) / (2 * h)
        out.append(num)
    return out


@pytest.mark.parametrize("nq,nk,causal,prefix", [(6, 6, False, 0), (7, 7, True, 0), (5, 9, True, 0), (9, 5, True, 0),
                                                  (4, 11, False, 0), (7, 7, True, 3), (5, 9, True, 6),
                                                  (9, 5, True, 2)])
def test_backward_matches_finite_differences(nq, nk, causal, prefix):
    # central differences of the (pinned) forward oracle: error O(h^2) ~ 1e-10 for h = 1e-5
    d, dv_, scale = 5, 4, 0.4
    rng = np.random.default_rng(nq * 31 + nk + 101 * prefix)
    q, k, v = rng.standard_normal((nq, d)), rng.standard_normal((nk, d)), rng.standard_normal((nk, dv_))
    do = rng.standard_normal((nq, dv_))
    grads = oracle.attention_head_backward(q, k, v, do, scale, causal, prefix)
    nums = _central_differences(lambda: _loss(q, k, v, do, scale, causal, prefix), (q, k, v))
    for g, num in zip(grads, nums):
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal,prefix", [(False, 0), (True, 0), (True, 4)])
def test_dense_backward_matches_finite_differences(causal, prefix):
    # the [B, N, H, D] layout: every (batch, head) differentiated with its own mask (prefix 4 widens
    # rows 0-2, which see keys 0..i+1 under the causal mask alone)
    B, nq, nk, H, d, scale = 2, 5, 6, 2, 3, 0.6
    rng = np.random.default_rng(23 + prefix + 7 * causal)
    q, do = rng.standard_normal((B, nq, H, d)), rng.standard_normal((B, nq, H, d))
    k, v = rng.standard_normal((B, nk, H, d)), rng.standard_normal((B, nk, H, d))

    def loss():
        o, _ = oracle.attention_dense(q, k, v, scale, causal, prefix)
        return float((o * do).sum())

    grads = oracle.attention_dense_backward(q, k, v, do, scale, causal, prefix)
    nums = _central_differences(loss, (q, k, v))
    for g, num in zip(grads, nums):
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal,prefix", [(False, 0), (True, 0), (True, 2)])
def test_varlen_backward_matches_finite_differences(causal, prefix):
    # packed sequences (one empty); the loss is taken over the packed forward oracle's output
    lengths, H, d, scale = [3, 0, 5, 1, 4], 2, 3, 0.7
    cu = si.cu_seqlens_of(lengths)
    total = int(cu[-1])
    rng = np.random.default_rng(17 + prefix + 5 * causal)
    q, k, v, do = (rng.standard_normal((total, H, d)) for _ in range(4))

    def loss():
        o, _ = oracle.attention_varlen(q, k, v, cu, scale, causal, prefix)
        return float((o * do).sum())

    grads = oracle.attention_varlen_backward(q, k, v, do, cu, scale, causal, prefix)
    nums = _central_differences(loss, (q, k, v))
    for g, num in zip(grads, nums):
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("nq,nk,causal,prefix,chunk", [(40, 40, False, 0, 7), (45, 45, True, 0, 8),
                                                        (30, 52, True, 0, 16), (52, 30, True, 0, 5),
                                                        (41, 41, True, 9, 6), (33, 50, False, 0, 64)])
def test_row_sampled_backward_matches_whole_head(nq, nk, causal, prefix, chunk):
    # every row and column sampled, query rows visited in blocks smaller than the head
    d, scale = 6, 0.35
    rng = np.random.default_rng(nq + 3 * nk + prefix)
    q, k, v, do = (rng.standard_normal(s) for s in ((nq, d), (nk, d), (nk, d), (nq, d)))
    dq, dk, dv = oracle.attention_head_backward(q, k, v, do, scale, causal, prefix)
    rows, cols = np.arange(nq)[::-1], np.arange(nk)[::-1]  # any order, returned in the order asked
    rq, rk, rv = oracle.attention_rows_backward(q, k, v, do, scale, rows, cols, causal, prefix, chunk=chunk)
    np.testing.assert_allclose(rq, dq[rows], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(rk, dk[cols], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(rv, dv[cols], rtol=1e-11, atol=1e-13)


def test_backward_closed_forms():
    # Q = 0, no mask: P is uniform 1/Nk, so dV_j = (1/Nk) sum_i dO_i for every key j and
    # dS_ij = (dO_i . V_j - dO_i . mean(V)) / Nk
    nq, nk, d = 6, 10, 4
    rng = np.random.default_rng(5)
    q = np.zeros((nq, d))
    k, v, do = rng.standard_normal((nk, d)), rng.standard_normal((nk, d)), rng.standard_normal((nq, d))
    dq, dk, dv = oracle.attention_head_backward(q, k, v, do, 0.5)
    np.testing.assert_allclose(dv, np.repeat(do.sum(axis=0, keepdims=True) / nk, nk, axis=0), rtol=1e-13)
    ds = (do @ v.T - (do @ v.mean(axis=0))[:, None]) / nk
    np.testing.assert_allclose(dq, 0.5 * ds @ k, rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(dk, np.zeros_like(k))  # dK = scale * dS^T Q = 0


def test_backward_row_sums_and_shift_invariance():
    # adding a vector c to every key shifts each score row by a constant, so P, dS and dV are
    # unchanged and dQ = scale dS (K + c) changes by scale (sum_j dS_ij) c = 0: dS rows sum to zero
    nq, nk, d = 8, 12, 5
    rng = np.random.default_rng(6)
    q, k, v, do = (rng.standard_normal(s) for s in ((nq, d), (nk, d), (nk, d), (nq, d)))
    dq, dk, dv = oracle.attention_head_backward(q, k, v, do, 0.3)
    c = rng.standard_normal(d)
    dq2, dk2, dv2 = oracle.attention_head_backward(q, k + c, v, do, 0.3)
    np.testing.assert_allclose(dq2, dq, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dv2, dv, rtol=1e-11, atol=1e-13)
    # total gradient wrt a key shift: sum_j dK_j = scale * sum_ij dS_ij q_i = 0
    np.testing.assert_allclose(dk.sum(axis=0), np.zeros(d), atol=1e-12)
