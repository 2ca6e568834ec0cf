"""Pins for the CPU oracle: each test fixes part of it against something other
than itself (a closed form, a library routine on a special case, brute force,
an invariant, or a hand-derived example).  CPU only.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import aqua_oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_orthogonal(d, seed):
    a = np.random.default_rng(seed).standard_normal((d, d))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))


def _std_attention(q, K, V, scale):
    """Textbook softmax attention of one query over keys K [T, d] (no projection, no selection)."""
    s = (K @ q) * scale
    w = np.exp(s - s.max())
    w /= w.sum()
    return w @ V


# --------------------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        np.array([1.0, -1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -7 + 2 ** -8, 2 ** -130, -2 ** -133,
                  3.3e38, 1e-45]),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_ties_and_no_double_rounding():
    # exact midpoints go to the even neighbour
    assert O.round_bf16(1 + 2 ** -8) == 1.0
    assert O.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6
    # just above a midpoint, by less than a float32 ulp: direct rounding goes up,
    # rounding through float32 would land on the midpoint and go to even (down)
    x = 1 + 2 ** -8 + 2 ** -30
    assert O.round_bf16(x) == 1 + 2 ** -7
    assert torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).item() == 1.0


# --------------------------------------------------------------------------- calibration

def test_calibrate_known_axes():
    # rows along scaled coordinate axes: right singular vectors are the axes,
    # ordered by the column norms 5 > 3 > 2 > 1
    X = np.zeros((8, 4))
    X[0, 2], X[1, 2] = 3.0, -4.0      # column 2 norm 5
    X[2, 0] = 3.0                      # column 0 norm 3
    X[3, 3], X[4, 3] = 2.0, 0.0        # column 3 norm 2
    X[5, 1] = -1.0                     # column 1 norm 1
    P, sigma = O.calibrate(X)
    np.testing.assert_allclose(sigma, [5, 3, 2, 1], atol=1e-12)
    np.testing.assert_allclose(np.abs(P), np.eye(4)[:, [2, 0, 3, 1]], atol=1e-12)


def test_calibrate_matches_gram_eigendecomposition():
    X = synth.calibration_matrix(n_q=2048, n_k=2048).astype(np.float64)
    P, sigma = O.calibrate(X)
    np.testing.assert_allclose(P.T @ P, np.eye(128), atol=1e-12)
    assert np.all(np.diff(sigma) <= 0)
    w, v = np.linalg.eigh(X.T @ X)          # a different routine on the same matrix
    w, v = w[::-1], v[:, ::-1]
    np.testing.assert_allclose(sigma ** 2, w, rtol=1e-9)
    # same columns up to sign
    dots = np.abs(np.sum(P * v, axis=0))
    np.testing.assert_allclose(dots, 1.0, atol=1e-8)


# --------------------------------------------------------------------------- selection

@pytest.mark.parametrize("seed", range(40))
def test_select_dims_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    d = int(rng.integers(2, 11))
    k = int(rng.integers(1, d + 1))
    m = int(rng.integers(k, d + 1))
    # small integers with repeats and +- pairs so ties are frequent
    qt = rng.integers(-3, 4, d).astype(np.float64)
    best, best_sum = None, -1.0
    for comb in itertools.combinations(range(m), k):   # lexicographic order
        s = float(np.sum(np.abs(qt[list(comb)])))
        if s > best_sum:
            best, best_sum = comb, s
    assert tuple(O.select_dims(qt, k, m)) == best


def test_select_identity_projection_is_raw_topk():
    # P = I: the projected query is the raw query; compare with a library sort
    rng = np.random.default_rng(3)
    q = rng.standard_normal(128)
    qt = O.project(q, np.eye(128))
    for k in (1, 32, 96, 128):
        ref = np.sort(np.argsort(-np.abs(q), kind="stable")[:k])
        np.testing.assert_array_equal(O.select_dims(qt, k), ref)


def test_attend_over_no_tokens_is_empty_sum():
    o, p, lse, S = O.attend_one(np.ones(8), 2, np.zeros((0, 8)), np.zeros((0, 8)), 1.0)
    assert np.all(o == 0) and p.size == 0 and lse == -np.inf and list(S) == [0, 1]


def test_select_rejects_bad_k():
    with pytest.raises(ValueError):
        O.select_dims(np.ones(8), 0)
    with pytest.raises(ValueError):
        O.select_dims(np.ones(8), 5, m=4)


# --------------------------------------------------------------------------- attention

def test_dense_k_equals_standard_attention():
    """k = d with an orthogonal P: q~.k~ = q P P^T k = q.k, so AQUA is standard attention."""
    d, T, Hq, Hkv = 128, 300, 4, 1
    P = _rand_orthogonal(d, 5)[None]
    q = synth.qk_tensor((1, Hq, d), 2)
    k = synth.qk_tensor((1, T, Hkv, d), 3)
    v = synth.v_tensor((1, T, Hkv, d), 4)
    Kt = O.build_key_cache(k, P, "f64").transpose(0, 2, 1, 3)
    V = v.transpose(0, 2, 1, 3)
    res = O.decode(q, P, Kt, V, [T], k=d)
    for h in range(Hq):
        ref = _std_attention(q[0, h].astype(np.float64), k[0, :, 0].astype(np.float64),
                             v[0, :, 0].astype(np.float64), 1 / math.sqrt(d))
        np.testing.assert_allclose(res["out"][0, h], ref, rtol=1e-11, atol=1e-12)


def test_dense_k_lse_equals_standard_logsumexp():
    """k = d with an orthogonal P: the step's log-sum-exp of the scaled scores is
    the textbook one over the raw q.k (closed form), computed here by scipy."""
    from scipy.special import logsumexp
    d, T, Hq = 128, 300, 4
    P = _rand_orthogonal(d, 7)[None]
    q = synth.qk_tensor((1, Hq, d), 2)
    k = synth.qk_tensor((1, T, 1, d), 3)
    v = synth.v_tensor((1, T, 1, d), 4)
    Kt = O.build_key_cache(k, P, "f64").transpose(0, 2, 1, 3)
    res = O.decode(q, P, Kt, v.transpose(0, 2, 1, 3), [T], k=d)
    for h in range(Hq):
        s = (k[0, :, 0].astype(np.float64) @ q[0, h].astype(np.float64)) / math.sqrt(d)
        assert abs(res["lse"][0, h] - logsumexp(s)) <= 1e-12 * max(1.0, abs(logsumexp(s)))
        np.testing.assert_allclose(np.sum(res["probs"][0][h]), 1.0, rtol=1e-13)


def test_dense_k_equals_standard_attention_fp32_cache():
    d, T = 128, 257
    P = _rand_orthogonal(d, 6)[None]
    q = synth.qk_tensor((1, 4, d), 2)
    k = synth.qk_tensor((1, T, 1, d), 3)
    v = synth.v_tensor((1, T, 1, d), 4)
    Kt = O.build_key_cache(k, P, "f32").transpose(0, 2, 1, 3)
    res = O.decode(q, P, Kt, v.transpose(0, 2, 1, 3), [T], k=d)
    for h in range(4):
        ref = _std_attention(q[0, h].astype(np.float64), k[0, :, 0].astype(np.float64),
                             v[0, :, 0].astype(np.float64), 1 / math.sqrt(d))
        err = np.linalg.norm(res["out"][0, h] - ref) / np.linalg.norm(ref)
        assert err <= 1e-5


def test_identity_projection_equals_masked_raw_attention():
    d, T, k = 128, 200, 64
    rng = np.random.default_rng(8)
    q = rng.standard_normal(d)
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    o, p, _, S = O.attend_one(O.project(q, np.eye(d)), k, K, V, 1 / math.sqrt(d))
    keep = np.argsort(-np.abs(q), kind="stable")[:k]
    qm = np.zeros(d)
    qm[keep] = q[keep]
    np.testing.assert_allclose(o, _std_attention(qm, K, V, 1 / math.sqrt(d)), rtol=1e-12, atol=1e-13)


def test_hadamard_golden():
    P = 0.5 * np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], dtype=np.float64)
    q = np.array([3.0, 1, 1, 1])
    K = np.array([[2.0, 0, 0, 0], [0, 2.0, 0, 0]])
    V = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0]])
    Kt = O.project(K, P)
    with open(os.path.join(GOLDEN, "hadamard_d4.txt")) as f:
        rows = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 3
    for ln in rows:
        left, right = ln.split("|")
        nums = [int(t) for t in left.split()]
        kk, sel = nums[0], nums[1:]
        o_ref = np.array([float(t) for t in right.split()])
        o, _, _, S = O.attend_one(O.project(q, P), kk, Kt, V, O.default_scale(4))
        assert list(S) == sel
        np.testing.assert_allclose(o, o_ref, rtol=1e-14, atol=1e-15)


def test_projection_sign_invariance():
    d, T = 128, 150
    P = _rand_orthogonal(d, 9)
    flip = np.where(np.random.default_rng(1).random(d) < 0.5, -1.0, 1.0)
    q = synth.qk_tensor((1, 4, d), 2)
    k = synth.qk_tensor((1, T, 1, d), 3)
    v = synth.v_tensor((1, T, 1, d), 4).transpose(0, 2, 1, 3)
    outs = []
    for PP in (P, P * flip[None, :]):
        Kt = O.build_key_cache(k, PP[None], "f64").transpose(0, 2, 1, 3)
        outs.append(O.decode(q, PP[None], Kt, v, [T], k=96))
    np.testing.assert_allclose(outs[0]["out"], outs[1]["out"], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(outs[0]["sel"], outs[1]["sel"])


def test_truncated_cache_matches_zero_tail_query():
    """m < d: a query whose projection is zero beyond m gives the same result
    with the truncated cache as with the full cache (selection never picks a zero)."""
    d, m, k, T = 128, 96, 64, 120
    P = _rand_orthogonal(d, 12)
    rng = np.random.default_rng(4)
    qt = rng.standard_normal(d)
    qt[m:] = 0.0
    q = qt @ P.T                       # so that q P = qt
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    Kt_full = O.project(K, P)
    o_full, _, _, S_full = O.attend_one(O.project(q, P), k, Kt_full, V, O.default_scale(d))
    o_trunc, _, _, S_tr = O.attend_one(O.project(q, P), k, Kt_full[:, :m], V, O.default_scale(d), m=m)
    np.testing.assert_array_equal(S_full, S_tr)
    np.testing.assert_allclose(o_full, o_trunc, rtol=1e-12, atol=1e-13)
    # m = d is the untruncated path
    o_md, _, _, _ = O.attend_one(O.project(q, P), k, Kt_full, V, O.default_scale(d), m=d)
    np.testing.assert_array_equal(o_md, o_full)


def test_truncated_cache_build_and_decode_keep_the_leading_dims():
    """The stored cache with m < d feeds a decode step that equals the full-cache
    step for queries whose projection vanishes beyond m (the leading m projected
    dimensions are the ones kept), and m = d is the untruncated cache."""
    d, m, k, T, Hq = 128, 96, 64, 90, 2
    P = _rand_orthogonal(d, 13)
    rng = np.random.default_rng(6)
    qt = rng.standard_normal((1, Hq, d))
    qt[..., m:] = 0.0
    q = qt @ P.T                                   # so that q P = qt
    kk = rng.standard_normal((1, T, 1, d))
    V = rng.standard_normal((1, 1, T, d))
    full = O.build_key_cache(kk, P[None], "f64").transpose(0, 2, 1, 3)
    trunc = O.build_key_cache(kk, P[None], "f64", m).transpose(0, 2, 1, 3)
    assert trunc.shape[-1] == m
    r_full = O.decode(q, P[None], full, V, [T], k)
    r_tr = O.decode(q, P[None], trunc, V, [T], k, m=m)
    np.testing.assert_array_equal(r_full["sel"], r_tr["sel"])
    np.testing.assert_allclose(r_tr["out"], r_full["out"], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(O.build_key_cache(kk, P[None], "f64", d), O.build_key_cache(kk, P[None], "f64"))


# --------------------------------------------------------------------------- value pruning (AQUA-Memory)

def _vp_case(seed, Hq=4, Hkv=2, T=50, d=128):
    rng = np.random.default_rng(seed)
    P = np.stack([_rand_orthogonal(d, seed + 1 + g) for g in range(Hkv)])
    q = rng.standard_normal((1, Hq, d))
    kk = rng.standard_normal((1, T, Hkv, d))
    vv = rng.standard_normal((1, T, Hkv, d))
    Kt = O.build_key_cache(kk, P, "f64").transpose(0, 2, 1, 3)
    return P, q, kk, vv, Kt


def _vp_decode(P, q, Kt, vv, m_v, k=64, store="f64"):
    Vh = O.build_value_cache(vv, P, store, m_v).transpose(0, 2, 1, 3)
    assert Vh.shape[-1] == m_v
    return O.decode(q, P, Kt, Vh, [vv.shape[1]], k, v_projected=True)


def test_value_pruning_at_full_width_is_the_unpruned_output():
    """m_v = d: V P P^T = V for orthogonal P, so projecting the values and
    bringing the output back changes nothing."""
    P, q, kk, vv, Kt = _vp_case(30)
    plain = O.decode(q, P, Kt, vv.transpose(0, 2, 1, 3), [vv.shape[1]], 64)
    pruned = _vp_decode(P, q, Kt, vv, 128)
    np.testing.assert_allclose(pruned["out"], plain["out"], rtol=1e-12, atol=1e-13)


def test_value_pruning_projects_the_output_onto_the_kept_subspace():
    """By linearity, pruning every value to the span of P's first m_v columns
    and summing equals summing first and projecting the unpruned output onto
    that span: o_pruned = o P_m P_m^T (computed here the other way round, from
    the unpruned decode).  The probabilities do not depend on the values."""
    P, q, kk, vv, Kt = _vp_case(31)
    plain = O.decode(q, P, Kt, vv.transpose(0, 2, 1, 3), [vv.shape[1]], 64)
    G = q.shape[1] // P.shape[0]
    for m_v in (96, 64, 1):
        pruned = _vp_decode(P, q, Kt, vv, m_v)
        for h in range(q.shape[1]):
            Pm = P[h // G][:, :m_v]
            expect = (plain["out"][0, h] @ Pm) @ Pm.T
            np.testing.assert_allclose(pruned["out"][0, h], expect, rtol=1e-11, atol=1e-12)
        np.testing.assert_array_equal(pruned["sel"], plain["sel"])
        np.testing.assert_allclose(pruned["lse"], plain["lse"], rtol=1e-14)


def test_value_pruning_sign_invariance():
    """Flipping the sign of columns of P flips the same stored value
    dimensions and their back-projection columns: the output is unchanged."""
    P, q, kk, vv, Kt = _vp_case(32)
    P2 = P.copy()
    P2[:, :, [0, 3, 70, 95, 100]] *= -1
    Kt2 = O.build_key_cache(kk, P2, "f64").transpose(0, 2, 1, 3)
    a = _vp_decode(P, q, Kt, vv, 96)
    b = _vp_decode(P2, q, Kt2, vv, 96)
    np.testing.assert_allclose(b["out"], a["out"], rtol=1e-12, atol=1e-13)


def test_value_pruning_is_lossless_for_values_in_the_kept_subspace():
    """Values built inside the span of each KV head's first m_v columns of P
    lose nothing: the pruned output equals the unpruned one."""
    P, q, kk, _, Kt = _vp_case(33)
    m_v = 80
    coeff = np.random.default_rng(34).standard_normal((1, kk.shape[1], P.shape[0], m_v))
    vv = np.einsum("btgj,gij->btgi", coeff, P[:, :, :m_v])
    plain = O.decode(q, P, Kt, vv.transpose(0, 2, 1, 3), [vv.shape[1]], 64)
    pruned = _vp_decode(P, q, Kt, vv, m_v)
    np.testing.assert_allclose(pruned["out"], plain["out"], rtol=1e-11, atol=1e-12)


def test_value_pruning_storage_rounds_the_projected_values():
    """bf16 storage: V^ is the RNE rounding of (v P)[:m_v] (not of v)."""
    P, q, kk, vv, Kt = _vp_case(35)
    Vh = O.build_value_cache(vv, P, "bf16", 96)
    exact = np.einsum("btgi,gij->btgj", vv, P)[..., :96]
    np.testing.assert_array_equal(Vh, O.round_bf16(exact))


def test_h2o_with_value_pruning():
    """H2O steps with pruned values: the evictions are those of plain H2O (they
    depend on the keys only) and every output is the plain output projected
    onto the kept value subspace; at m_v = d the outputs are the plain ones."""
    d, Hq, Hkv, n0, k = 128, 4, 2, 12, 48
    rng = np.random.default_rng(36)
    P = np.stack([_rand_orthogonal(d, 37 + g) for g in range(Hkv)])
    kk = rng.standard_normal((n0 + 6, Hkv, d))
    vv = rng.standard_normal((n0 + 6, Hkv, d))
    q = rng.standard_normal((6, Hq, d))
    for m_v in (96, 128):
        def seqs(project_v):
            return [O.H2OSeq(pos=list(range(n0)), score=[0.0] * n0,
                             kt=list(O.build_key_cache(kk[:n0, g][:, None], P[g][None], "f64")[:, 0]),
                             v=list(O.build_value_cache(vv[:n0, g][:, None], P[g][None], "f64", m_v)[:, 0])
                             if project_v else list(vv[:n0, g]))
                    for g in range(Hkv)]
        a, b = seqs(False), seqs(True)
        for s in range(6):
            oa, ea = O.h2o_decode_step(a, q[s], kk[n0 + s], vv[n0 + s], n0 + s, P, k, 14, 3, "f64")
            ob, eb = O.h2o_decode_step(b, q[s], kk[n0 + s], vv[n0 + s], n0 + s, P, k, 14, 3, "f64", m_v=m_v)
            assert ea == eb
            for h in range(Hq):
                Pm = P[h // (Hq // Hkv)][:, :m_v]
                np.testing.assert_allclose(ob[h], (oa[h] @ Pm) @ Pm.T, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------- prefill vs decode

def test_prefill_row_equals_decode_and_chunk_invariance():
    d, Hq, Hkv, L, k = 128, 4, 2, 24, 96
    P = np.stack([_rand_orthogonal(d, 20), _rand_orthogonal(d, 21)])
    inp = synth.prefill_inputs(L, Hq, Hkv, bf16=True)
    Kt = O.build_key_cache(inp["k"][0], P, "bf16").transpose(1, 0, 2)    # [Hkv, L, d]
    V = inp["v"][0].transpose(1, 0, 2)
    out_all, sel_all = O.prefill(inp["q"][0], 0, P, Kt, V, k)
    # chunk-size invariance: 3 chunks of 8 rows
    parts = [O.prefill(inp["q"][0][c:c + 8], c, P, Kt, V, k)[0] for c in (0, 8, 16)]
    np.testing.assert_allclose(np.concatenate(parts), out_all, rtol=1e-13, atol=1e-14)
    # row p equals a decode step that sees tokens 0..p
    for p in (0, 7, 23):
        res = O.decode(inp["q"][0][p][None], P, Kt[None], V[None], [p + 1], k)
        np.testing.assert_allclose(res["out"][0], out_all[p], rtol=1e-13, atol=1e-14)
        np.testing.assert_array_equal(res["sel"][0], sel_all[p])


# --------------------------------------------------------------------------- H2O

def _h2o_run(budget, recent, steps, T0, k=64, m=None, seed_shift=0):
    d, Hq, Hkv = 128, 4, 2
    P = np.stack([_rand_orthogonal(d, 30), _rand_orthogonal(d, 31)])
    inp = synth.decode_inputs(1, Hq, Hkv, T0, bf16=True, steps=steps)
    seqs = []
    for g in range(Hkv):
        kt = O.build_key_cache(inp["k_hist"][0, :, g][:, None], P[g][None], "bf16", m)[:, 0]
        seqs.append(O.H2OSeq(pos=list(range(T0)), score=[0.0] * T0, kt=list(kt),
                             v=list(inp["v_hist"][0, :, g].astype(np.float64))))
    outs, evs = [], []
    for s in range(steps):
        o, ev = O.h2o_decode_step(seqs, inp["q"][s, 0], inp["k_new"][s, 0], inp["v_new"][s, 0], T0 + s,
                                  P, k, budget, recent, "bf16", m)
        outs.append(o)
        evs.append(ev)
    return P, inp, seqs, outs, evs


def test_h2o_large_budget_is_plain_decode():
    T0, steps = 40, 5
    P, inp, seqs, outs, evs = _h2o_run(budget=1000, recent=8, steps=steps, T0=T0)
    assert all(e == -1 for ev in evs for e in ev)
    k_all = np.concatenate([inp["k_hist"], inp["k_new"].transpose(1, 0, 2, 3)], axis=1)
    v_all = np.concatenate([inp["v_hist"], inp["v_new"].transpose(1, 0, 2, 3)], axis=1)
    Kt = O.build_key_cache(k_all, P, "bf16").transpose(0, 2, 1, 3)
    for s in range(steps):
        res = O.decode(inp["q"][s], P, Kt, v_all.transpose(0, 2, 1, 3), [T0 + s + 1], 64)
        np.testing.assert_allclose(outs[s], res["out"][0], rtol=1e-12, atol=1e-13)


def test_h2o_cumulative_score_is_sum_of_group_probabilities():
    """With no eviction, a token's cumulative score after the last step is the
    sum, over every step since it entered and over the group's query heads, of
    its softmax probability in a plain decode step over the same tokens."""
    T0, steps, G = 30, 4, 2
    P, inp, seqs, outs, evs = _h2o_run(budget=1000, recent=8, steps=steps, T0=T0)
    k_all = np.concatenate([inp["k_hist"], inp["k_new"].transpose(1, 0, 2, 3)], axis=1)
    v_all = np.concatenate([inp["v_hist"], inp["v_new"].transpose(1, 0, 2, 3)], axis=1)
    Kt = O.build_key_cache(k_all, P, "bf16").transpose(0, 2, 1, 3)
    acc = np.zeros((2, T0 + steps))
    for s in range(steps):
        res = O.decode(inp["q"][s], P, Kt, v_all.transpose(0, 2, 1, 3), [T0 + s + 1], 64)
        for h in range(4):
            acc[h // G, :T0 + s + 1] += res["probs"][0][h]
    for g in range(2):
        assert seqs[g].pos == list(range(T0 + steps))
        np.testing.assert_allclose(seqs[g].score, acc[g], rtol=1e-12, atol=1e-15)


def test_h2o_recent_equals_budget_is_sliding_window():
    T0, budget, steps = 16, 16, 6
    P, inp, seqs, outs, evs = _h2o_run(budget=budget, recent=budget, steps=steps, T0=T0)
    for s in range(steps):
        assert evs[s] == [s, s]            # the oldest position leaves each step
    for g in range(2):
        assert seqs[g].pos == list(range(T0 + steps - budget, T0 + steps))
    # attention runs after the append and before the eviction, so each step
    # sees the last budget + 1 tokens
    k_all = np.concatenate([inp["k_hist"], inp["k_new"].transpose(1, 0, 2, 3)], axis=1)
    v_all = np.concatenate([inp["v_hist"], inp["v_new"].transpose(1, 0, 2, 3)], axis=1)
    Kt = O.build_key_cache(k_all, P, "bf16").transpose(0, 2, 1, 3)
    V = v_all.transpose(0, 2, 1, 3)
    for s in range(steps):
        lo, hi = T0 + s - budget, T0 + s + 1
        res = O.decode(inp["q"][s], P, Kt[:, :, lo:hi], V[:, :, lo:hi], [budget + 1], 64)
        np.testing.assert_allclose(outs[s], res["out"][0], rtol=1e-12, atol=1e-13)


def test_h2o_victim_rule_hand_case():
    # positions 10..15, newest 15, recent 2 -> 14, 15 protected
    pos = [10, 11, 12, 13, 14, 15]
    score = [0.5, 0.2, 0.2, 0.9, 0.0, 0.0]
    assert O.h2o_choose_victim(score, pos, 15, 2) == 1          # tie 0.2: older position 11
    assert O.h2o_choose_victim(score, [12, 11, 10, 13, 14, 15], 15, 2) == 2   # tie: position 10 is older
    assert O.h2o_choose_victim([0.0] * 3, [5, 6, 7], 7, 3) == -1  # everything is recent


# --------------------------------------------------------------------------- magnitude vs slicing

def test_query_energy_loss_hand_values():
    qt = np.array([3.0, 4.0, 0.0, 0.0])                 # |q|^2 = 25
    assert O.query_energy_loss(qt, [1]) == pytest.approx(1 - 16 / 25)
    assert O.query_energy_loss(qt, [0]) == pytest.approx(1 - 9 / 25)
    assert O.query_energy_loss(qt, [0, 1]) == 0.0
    assert O.query_energy_loss(qt, [2, 3]) == 1.0
    assert O.query_energy_loss(np.zeros(4), [0]) == 0.0


@pytest.mark.parametrize("seed", range(6))
def test_magnitude_selection_minimises_the_energy_loss(seed):
    """Brute force over every k-subset of a tiny projected query: the k largest
    magnitudes lose the least squared norm."""
    rng = np.random.default_rng(100 + seed)
    d = 8
    qt = rng.standard_normal(d)
    for k in range(1, d + 1):
        best = min(O.query_energy_loss(qt, list(S)) for S in itertools.combinations(range(d), k))
        assert O.query_energy_loss(qt, O.select_dims(qt, k)) == pytest.approx(best, abs=1e-15)


def test_attention_output_loss_hand_case():
    """Two tokens with one-hot keys and values, scale 1: full scores (ln 3, ln 2)
    give o = (3/5, 2/5); keeping dimension 0 only gives scores (ln 3, 0) and
    o_S = (3/4, 1/4); the loss is |o_S - o| / |o| = 0.15 sqrt(2) / sqrt(0.52)."""
    qt = np.array([np.log(3.0), np.log(2.0)])
    Kt = np.eye(2)
    V = np.eye(2)
    got = O.attention_output_loss(qt, [0], Kt, V, 1.0)
    assert got == pytest.approx(0.15 * np.sqrt(2) / np.sqrt(0.52), rel=1e-12)
    assert O.attention_output_loss(qt, [0, 1], Kt, V, 1.0) == 0.0


def test_slicing_is_the_leading_block_and_equals_magnitude_when_sorted():
    assert list(O.select_first_dims(3, 8)) == [0, 1, 2]
    d, k = 16, 6
    rng = np.random.default_rng(7)
    q = np.sort(np.abs(rng.standard_normal((3, d))), axis=1)[:, ::-1] * rng.choice([-1, 1], (3, d))
    K = rng.standard_normal((20, d))
    V = rng.standard_normal((20, d))
    r = O.retention_losses(q, np.eye(d), K, V, k)
    assert r["magnitude"] == r["slicing"]          # the largest magnitudes are the first dims


def test_retention_losses_use_the_projected_query():
    """With P a permutation that moves the query's large entries to the end of
    the projected space, magnitude selection (on q~ = q P) keeps them and loses
    nothing of the energy, while slicing the first k projected dims loses it all."""
    d, k = 8, 2
    perm = np.roll(np.eye(d), 6, axis=1)              # q~_j = q_(j - 6 mod 8): q_0, q_1 -> dims 6, 7
    q = np.zeros((1, d))
    q[0, :2] = [5.0, -4.0]
    rng = np.random.default_rng(8)
    K = rng.standard_normal((12, d))
    V = rng.standard_normal((12, d))
    qt = O.project(q[0], perm)
    assert list(np.nonzero(qt)[0]) == [6, 7]
    r = O.retention_losses(q, perm, K, V, k)
    assert r["magnitude"]["energy"] == 0.0 and r["magnitude"]["output"] == pytest.approx(0.0, abs=1e-15)
    assert r["slicing"]["energy"] == 1.0 and r["slicing"]["output"] > 0.0


# --------------------------------------------------------------------------- counts

def test_qk_mac_count_matches_pages_25_percent():
    # the pages' figure: a 25% cut of the attention dot-product work at k = 96 of d = 128
    T = 8192
    assert O.qk_macs(T, 128, 96) / O.qk_macs(T, 128) == 0.75


class _MacCounter(np.ndarray):
    """ndarray that adds the multiply-adds of every matmul it takes part in to
    a shared tally (output elements times the contracted length)."""
    tally = [0]

    def __array_ufunc__(self, ufunc, method, *inputs, **kw):
        args = [np.asarray(x) if isinstance(x, _MacCounter) else x for x in inputs]
        res = getattr(ufunc, method)(*args, **kw)
        if ufunc is np.matmul and method == "__call__":
            _MacCounter.tally[0] += int(np.prod(np.shape(res))) * args[0].shape[-1]
        return res.view(_MacCounter) if isinstance(res, np.ndarray) else res


class _NumpyKeepingSubclasses:
    """Stand-in for the oracle module's numpy whose asarray keeps array
    subclasses (so the counter survives the oracle's input conversions)."""

    def __getattr__(self, name):
        return getattr(np, name)

    @staticmethod
    def asarray(a, dtype=None):
        return np.asanyarray(a, dtype=dtype)


def _counted_macs(fn):
    _MacCounter.tally[0] = 0
    fn()
    return _MacCounter.tally[0]


def test_breakeven_matches_the_oracles_own_operation_count():
    """The break-even length is the first context length at which one AQUA
    decode step costs fewer multiply-adds than dense attention, per query
    head.  Both costs are COUNTED here on the oracle's own functions (every
    matmul they execute, through a counting array type), not recomputed from
    a formula: AQUA = the query projection + 1/G of the key projection (one
    new key per KV head serves its G query heads) + the scores on the k
    selected dimensions; dense = the textbook q . k over all d dimensions.
    A search over T finds the first T where AQUA is cheaper; breakeven_length
    must agree with it to within one token."""
    saved = O.np
    O.np = _NumpyKeepingSubclasses()
    try:
        _breakeven_search()
    finally:
        O.np = saved


def _breakeven_search():
    d = 128
    rng = np.random.default_rng(3)
    P = _rand_orthogonal(d, 4).view(_MacCounter)
    K_all = rng.standard_normal((8192, d)).view(_MacCounter)
    q = rng.standard_normal(d).view(_MacCounter)
    k_new = rng.standard_normal(d).view(_MacCounter)
    for k, G in [(96, 4), (64, 4), (32, 4), (96, 1), (120, 2), (64, 2)]:
        def aqua(T):
            def step():
                qt = O.project(q, P)
                S = O.select_dims(np.asarray(qt), k)
                O.sparse_scores(qt, S, K_all[:T], 1.0)
            kproj = _counted_macs(lambda: O.project(k_new, P))
            return _counted_macs(step) + kproj / G

        def dense(T):
            return _counted_macs(lambda: K_all[:T] @ q)

        assert aqua(1000) - aqua(999) == k and dense(1000) - dense(999) == d   # k, d per token
        lo, hi = 1, 8192
        assert aqua(hi) < dense(hi) and not aqua(lo) < dense(lo)
        while hi - lo > 1:                 # first T with aqua(T) < dense(T) is hi
            mid = (lo + hi) // 2
            if aqua(mid) < dense(mid):
                hi = mid
            else:
                lo = mid
        T_star = O.breakeven_length(d, k, G)
        assert abs(hi - T_star) <= 1, (k, G, hi, T_star)
    assert O.breakeven_length(d, d, 4) == float("inf")   # no saving per token: no break-even
