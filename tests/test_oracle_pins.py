"""Pins for the fp64 oracle: each check compares the oracle with something other
than itself -- hand-derived closed forms, brute force on tiny inputs, an
independent library routine for a special case, or an invariant of the
definition -- so that a dropped term, a wrong index or a transposed operand in
oracle/ fails here.

Method definition: "Loki: Low-rank Keys for Efficient Sparse Attention"
(atlas.scime.ai summary), sections "Approach" and the summary paragraph.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import get_workload
from workloads import generators as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _scale(s):
    return {"ln3": math.log(3.0), "ln2/3": math.log(2.0) / 3.0}[s]


def _hand_case(name):
    c = _load(name)
    P = np.array(c["P"], dtype=np.float64)
    q = np.array(c["q"], dtype=np.float64)
    keys = np.array(c["keys"], dtype=np.float64)
    vals = np.array(c["values"], dtype=np.float64)
    K_hat = oracle.rotate_keys(keys, P, "f64")
    return c, P, q, K_hat, vals


# ---------------------------------------------------------------- hand cases
@pytest.mark.parametrize("name", ["hand_2d_swap.json", "hand_gqa_sum.json"])
def test_hand_cases(name):
    c, P, q, K_hat, vals = _hand_case(name)
    r = oracle.loki_decode(q, K_hat, vals, P, c["S"], c["d"], c["k"], scale=_scale(c["scale"]))
    np.testing.assert_allclose(r["scores"], np.array(c["expected_scores"]), rtol=0, atol=1e-15)
    assert r["idx"].tolist() == c["expected_idx"]
    np.testing.assert_allclose(r["out"], np.array(c["expected_out"]), rtol=0, atol=1e-14)


def test_hand_2d_swap_default_scale():
    c, P, q, K_hat, vals = _hand_case("hand_2d_swap.json")
    r = oracle.loki_decode(q, K_hat, vals, P, 4, 1, 2)  # default scale 1/sqrt(D)
    w1 = 1.0 / (1.0 + math.exp(1.0 / math.sqrt(2.0)))
    w3 = 1.0 - w1
    np.testing.assert_allclose(r["out"][0, 0], [4.0 * w1, 8.0 * w3], rtol=0, atol=1e-14)


# ---------------------------------------------------------------- rounding
def test_round_bf16_matches_torch_on_fp32_inputs():
    # torch's fp32 -> bf16 cast rounds to nearest even; on fp32-representable
    # inputs a single rounding from fp64 must agree with it exactly.
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        rng.standard_normal(2000) * 1e-39,                     # bf16 subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-45]),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_ties_and_overflow():
    # 1 + 2^-8 is exactly halfway between 1 and 1 + 2^-7: ties go to the even
    # significand (1.0); 1 + 3*2^-8 is halfway between 1+2^-7 and 1+2^-6 -> 1+2^-6.
    assert oracle.round_bf16(1.0 + 2.0 ** -8) == 1.0
    assert oracle.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert oracle.round_bf16(-(1.0 + 2.0 ** -8)) == -1.0
    # just above halfway rounds up
    assert oracle.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
    # the largest finite bf16 plus half an ulp overflows; slightly less does not
    mx = oracle.BF16_MAX
    assert np.isinf(oracle.round_bf16(mx + 2.0 ** 119))
    assert oracle.round_bf16(mx + 2.0 ** 118) == mx
    # not representable in fp32 either: fp64 value between two bf16 values that
    # a double rounding through fp32 would send the wrong way
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40      # fp32 rounds this to 1 + 2^-8 (a tie), then to 1.0
    assert oracle.round_bf16(x) == 1.0 + 2.0 ** -7


def test_round_f32_is_numpy_cast():
    x = np.array([1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, 0.1])
    np.testing.assert_array_equal(oracle.round_to_dtype(x, "f32"),
                                  np.array([1.0, 1.0 + 2.0 ** -22, np.float32(0.1)], dtype=np.float64))


# ---------------------------------------------------------------- PCA
def test_pca_closed_form_axis_aligned():
    # keys +-a_j e_j: mean 0, covariance exactly diag(a_j^2 * 2/N) -> P is the
    # permutation that sorts a_j descending, every column with a +1 entry.
    D = 6
    a = np.array([1.0, 5.0, 2.0, 4.0, 3.0, 0.5])
    X = []
    for j in range(D):
        e = np.zeros(D)
        e[j] = a[j]
        X += [e, -e]
    P, w = oracle.pca_basis(np.array(X))
    order = np.argsort(-a)
    np.testing.assert_allclose(P, np.eye(D)[:, order], atol=1e-12)
    np.testing.assert_allclose(w, a[order] ** 2 * 2 / (2 * D), rtol=1e-12)


def test_pca_closed_form_2d_rotation():
    # variance 9 along (cos t, sin t) and 1 along (-sin t, cos t)
    t = 0.3
    d1 = np.array([math.cos(t), math.sin(t)])
    d2 = np.array([-math.sin(t), math.cos(t)])
    X = np.array([3 * d1, -3 * d1, d2, -d2]) * math.sqrt(2.0)
    P, w = oracle.pca_basis(X)
    np.testing.assert_allclose(w, [9.0, 1.0], rtol=1e-12)
    np.testing.assert_allclose(P[:, 0], d1, atol=1e-12)       # largest entry cos t > 0
    np.testing.assert_allclose(P[:, 1], d2, atol=1e-12)       # largest entry cos t > 0


@pytest.mark.parametrize("wname", ["tiny-fp32", "llama2-7b-decode"])
def test_pca_definition_on_workload(wname):
    w = get_workload(wname)
    X = gen.calibration_keys(w, 0)
    P, lam = oracle.pca_basis(X)
    Xc = X - X.mean(0)
    C = Xc.T @ Xc / X.shape[0]
    D = w.head_dim
    np.testing.assert_allclose(P.T @ P, np.eye(D), atol=1e-12)          # orthonormal
    np.testing.assert_allclose(C @ P, P * lam[None, :], atol=1e-10)      # C P = P Lambda
    assert np.all(np.diff(lam) <= 1e-12)                                  # descending
    lead = np.argmax(np.abs(P), axis=0)
    assert np.all(P[lead, np.arange(D)] > 0)                              # sign rule
    # independent eigen-solver agrees on the spectrum
    np.testing.assert_allclose(lam, np.sort(np.linalg.eigvalsh(C))[::-1], rtol=1e-9, atol=1e-12)
    if w.generator == "rank8":
        # rank 8 plus 0.05 noise: 8 large eigenvalues; the other D-8 are the
        # noise variance 0.05^2 spread over the Marchenko-Pastur support
        # 0.0025 * (1 -+ sqrt(gamma))^2 with gamma = (D-8)/N
        assert lam[7] > 1.0
        noise = lam[8:]
        gam = (D - 8) / X.shape[0]
        lo, hi = 0.0025 * (1 - math.sqrt(gam)) ** 2, 0.0025 * (1 + math.sqrt(gam)) ** 2
        assert abs(noise.mean() - 0.0025) < 0.05 * 0.0025
        assert noise.min() > 0.8 * lo and noise.max() < 1.2 * hi
    else:
        # the sample spectrum follows the generating power law
        lam_true = gen.power_law_spectrum(D, w.alpha)
        np.testing.assert_allclose(lam[:8], lam_true[:8], rtol=0.12)


def test_pca_recovers_generating_basis():
    # with many samples the leading principal directions match the columns of
    # the generator's orthonormal U up to sign
    w = get_workload("llama2-7b-decode").with_(n_calib=40000)
    m = gen.make_key_model(w, 3)
    X = gen.draw_keys(m, w.n_calib, np.random.default_rng(11))
    P, _ = oracle.pca_basis(X)
    for j in range(3):
        assert abs(abs(P[:, j] @ m.U[:, j]) - 1.0) < 2e-3


# ---------------------------------------------------------------- rotation
def test_rotation_preserves_full_dot_products():
    rng = np.random.default_rng(3)
    D = 64
    P, _ = oracle.pca_basis(rng.standard_normal((500, D)) @ rng.standard_normal((D, D)))
    q = rng.standard_normal((1, 1, D))
    k = rng.standard_normal((1, 1, 50, D))
    q_hat = oracle.rotate_queries(q, P[None])
    k_hat = oracle.rotate_keys(k, P[None], "f64")
    np.testing.assert_allclose(k_hat[0, 0] @ q_hat[0, 0], k[0, 0] @ q[0, 0], rtol=1e-12, atol=1e-12)


def test_rotate_keys_identity_and_permutation():
    rng = np.random.default_rng(4)
    k = rng.standard_normal((2, 3, 5, 8))
    eye = np.broadcast_to(np.eye(8), (3, 8, 8))
    np.testing.assert_array_equal(oracle.rotate_keys(k, eye, "f64"), k)
    np.testing.assert_array_equal(oracle.rotate_keys(k, eye, "bf16"), oracle.round_bf16(k))
    perm = np.eye(8)[:, ::-1]           # column j = e_{7-j}: reverses coordinates
    Pm = np.broadcast_to(perm, (3, 8, 8))
    np.testing.assert_array_equal(oracle.rotate_keys(k, Pm, "f64"), k[..., ::-1])
    # a different P per KV head is applied to its own head only
    P2 = np.stack([np.eye(8), perm, 2 * np.eye(8)])
    r = oracle.rotate_keys(k, P2, "f64")
    np.testing.assert_array_equal(r[:, 0], k[:, 0])
    np.testing.assert_array_equal(r[:, 1], k[:, 1, :, ::-1])
    np.testing.assert_array_equal(r[:, 2], 2 * k[:, 2])


def test_append_writes_only_new_positions():
    rng = np.random.default_rng(5)
    B, H, Scap, D = 2, 2, 10, 4
    K = np.full((B, H, Scap, D), 7.0)
    V = np.full((B, H, Scap, D), 9.0)
    kn = rng.standard_normal((B, H, 3, D))
    vn = rng.standard_normal((B, H, 3, D))
    P = np.broadcast_to(np.eye(D), (H, D, D))
    oracle.append(K, V, 4, kn, vn, P, "f32")
    assert np.all(K[:, :, :4] == 7.0) and np.all(K[:, :, 7:] == 7.0)
    np.testing.assert_array_equal(K[:, :, 4:7], kn.astype(np.float32).astype(np.float64))
    np.testing.assert_array_equal(V[:, :, 4:7], vn)


# ---------------------------------------------------------------- top-k
def _brute_topk(s, k):
    # token i is selected iff fewer than k tokens rank before it, where j ranks
    # before i when s_j > s_i, or s_j == s_i and j < i.  O(S^2), no sorting.
    S = len(s)
    sel = []
    for i in range(S):
        before = sum(1 for j in range(S) if s[j] > s[i] or (s[j] == s[i] and j < i))
        if before < k:
            sel.append(i)
    return sel


@pytest.mark.parametrize("seed", range(20))
def test_topk_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    S = int(rng.integers(1, 40))
    s = rng.integers(-4, 5, S).astype(np.float64)       # heavy ties
    if seed % 3 == 0:
        s = rng.standard_normal(S)
    for k in sorted({1, max(1, S // 2), S}):
        assert oracle.select_topk(s[None], k)[0].tolist() == _brute_topk(s, k)


def test_topk_matches_torch_on_distinct_scores():
    rng = np.random.default_rng(9)
    s = rng.standard_normal((6, 1000))
    k = 137
    got = oracle.select_topk(s, k)
    ref = torch.topk(torch.from_numpy(s), k, dim=-1).indices.sort(dim=-1).values.numpy()
    np.testing.assert_array_equal(got, ref)


def test_topk_negative_zero_ties_positive_zero():
    s = np.array([0.0, -0.0, 0.0, -0.0, -1.0])
    assert oracle.select_topk(s[None], 3)[0].tolist() == [0, 1, 2]


# ---------------------------------------------------------------- decode
def _rand_case(seed, B=2, Hq=4, Hkv=2, D=16, S=40, dtype="f64"):
    rng = np.random.default_rng(seed)
    P = np.stack([oracle.pca_basis(rng.standard_normal((200, D)) @ rng.standard_normal((D, D)))[0]
                  for _ in range(Hkv)])
    q = rng.standard_normal((B, Hq, D))
    keys = rng.standard_normal((B, Hkv, S, D))
    V = rng.standard_normal((B, Hkv, S, D))
    K_hat = oracle.rotate_keys(keys, P, dtype)
    return P, q, keys, K_hat, V


def _sdpa_reference(q, keys, V, S, scale):
    # torch's scaled_dot_product_attention in fp64 on the UNROTATED keys,
    # GQA heads expanded to their KV head
    B, Hq, D = q.shape
    Hkv = keys.shape[1]
    G = Hq // Hkv
    qt = torch.from_numpy(q)[:, :, None, :]
    kt = torch.from_numpy(np.repeat(keys[:, :, :S], G, axis=1))
    vt = torch.from_numpy(np.repeat(V[:, :, :S], G, axis=1))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o[:, :, 0, :].numpy()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_full_budget_is_dense_attention(seed):
    # d = D and k = S keep every token: Loki reduces to exact attention, and an
    # orthonormal P cancels between q and k.
    P, q, keys, K_hat, V = _rand_case(seed)
    D, S = q.shape[-1], 40
    r = oracle.loki_decode(q, K_hat, V, P, S, D, S)
    ref = _sdpa_reference(q, keys, V, S, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.dense_decode(q, K_hat, V, P, S), ref, rtol=0, atol=1e-12)
    assert np.all(r["idx"] == np.arange(S))


def test_dense_attends_only_first_seq_len_tokens():
    P, q, keys, K_hat, V = _rand_case(5, S=40)
    K_hat[:, :, 30:] = 1e6          # garbage beyond seq_len must not matter
    V[:, :, 30:] = np.nan
    ref = _sdpa_reference(q, keys, V, 30, 0.25)
    np.testing.assert_allclose(oracle.dense_decode(q, K_hat, V, P, 30, scale=0.25), ref, atol=1e-12)
    r = oracle.loki_decode(q, K_hat, V, P, 30, 16, 30, scale=0.25)
    np.testing.assert_allclose(r["out"], ref, atol=1e-12)


def test_softmax_weights_sum_to_one():
    P, q, keys, K_hat, V = _rand_case(6)
    r = oracle.loki_decode(q, K_hat, V, P, 40, 4, 13)
    np.testing.assert_allclose(r["weights"].sum(-1), 1.0, rtol=0, atol=1e-15)
    assert np.all(r["weights"] > 0)


def test_k1_returns_value_of_best_token():
    P, q, keys, K_hat, V = _rand_case(7, Hq=2, Hkv=2)
    r = oracle.loki_decode(q, K_hat, V, P, 40, 5, 1)
    for b in range(2):
        for g in range(2):
            best = int(np.argmax(r["scores"][b, g]))
            assert r["idx"][b, g, 0] == best
            np.testing.assert_array_equal(r["out"][b, g], V[b, g, best])


def test_zero_query_ties_take_lowest_indices():
    P, q, keys, K_hat, V = _rand_case(8)
    q[:] = 0.0
    r = oracle.loki_decode(q, K_hat, V, P, 40, 8, 11)
    assert np.all(r["idx"] == np.arange(11))
    # all logits equal -> uniform weights -> mean of the first k values
    G = 2
    for h in range(4):
        np.testing.assert_allclose(r["out"][:, h], V[:, h // G, :11].mean(axis=1), atol=1e-15)


def test_gqa_score_is_linear_in_group_queries():
    P, q, keys, K_hat, V = _rand_case(9, Hq=8, Hkv=2)
    d = 6
    r = oracle.loki_decode(q, K_hat, V, P, 40, d, 10)
    q_hat = oracle.rotate_queries(q, P)
    for b in range(2):
        for g in range(2):
            u = q_hat[b, 4 * g:4 * g + 4, :d].sum(axis=0)
            np.testing.assert_allclose(r["scores"][b, g], K_hat[b, g, :, :d] @ u, rtol=1e-12, atol=1e-12)


def test_gqa_identical_heads_select_like_one_head():
    P, q, keys, K_hat, V = _rand_case(10, Hq=4, Hkv=1)
    q[:, 1:] = q[:, :1]
    r4 = oracle.loki_decode(q, K_hat, V, P, 40, 5, 9)
    r1 = oracle.loki_decode(q[:, :1], K_hat, V, P, 40, 5, 9)
    np.testing.assert_array_equal(r4["idx"], r1["idx"])
    np.testing.assert_allclose(r4["out"][:, 0], r1["out"][:, 0], atol=1e-15)


def test_selection_uses_first_d_principal_dims():
    # rank-r keys (r <= d), no noise, P calibrated on the same distribution:
    # every key lies in the span of the first r principal directions, so the
    # low-rank ranking equals the full-dimension ranking (exact top-k).
    rng = np.random.default_rng(12)
    D, r, S = 32, 4, 200
    A = rng.standard_normal((r, D))
    calib = rng.standard_normal((2000, r)) @ A
    P, lam = oracle.pca_basis(calib)
    assert lam[r] < 1e-12 * lam[0]
    keys = (rng.standard_normal((S, r)) @ A)[None, None]
    K_hat = oracle.rotate_keys(keys, P[None], "f64")
    q = rng.standard_normal((1, 1, D))
    for d in (r, r + 3, 16):
        lo = oracle.loki_decode(q, K_hat, keys * 0, P[None], S, d, 50)["idx"]
        ex = oracle.loki_decode(q, K_hat, keys * 0, P[None], S, D, 50)["idx"]
        np.testing.assert_array_equal(lo, ex)
    # with d < r the ranking generally differs (the pin can fail)
    lo = oracle.loki_decode(q, K_hat, keys * 0, P[None], S, 1, 50)["idx"]
    assert not np.array_equal(lo, ex)


def test_selection_invariant_to_key_shift_and_query_scale():
    P, q, keys, K_hat, V = _rand_case(13)
    d, k = 5, 12
    r0 = oracle.loki_decode(q, K_hat, V, P, 40, d, k)
    # a constant added to every key shifts every score of a row by the same amount
    c = np.random.default_rng(0).standard_normal(16)
    K_shift = oracle.rotate_keys(keys + c, P, "f64")
    r1 = oracle.loki_decode(q, K_shift, V, P, 40, d, k)
    np.testing.assert_array_equal(r0["idx"], r1["idx"])
    # a positive query scale scales every score
    r2 = oracle.loki_decode(3.5 * q, K_hat, V, P, 40, d, k)
    np.testing.assert_array_equal(r0["idx"], r2["idx"])


def test_sign_flip_of_basis_column_changes_nothing():
    # eigenvector signs are arbitrary: flipping column j flips coordinate j of
    # both q_hat and k_hat, leaving scores and outputs unchanged
    P, q, keys, K_hat, V = _rand_case(14)
    P2 = P.copy()
    P2[:, :, 2] *= -1
    K2 = oracle.rotate_keys(keys, P2, "f64")
    a = oracle.loki_decode(q, K_hat, V, P, 40, 6, 10)
    b = oracle.loki_decode(q, K2, V, P2, 40, 6, 10)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_allclose(a["out"], b["out"], atol=1e-13)


# ---------------------------------------------------------------- drift guard
def test_oracle_matches_stored_tiny_output():
    # the stored file was written by tests/golden/make_oracle_golden.py, which
    # calls only the oracle; a change of oracle arithmetic shows up here
    import importlib.util
    spec = importlib.util.spec_from_file_location("mk", os.path.join(GOLDEN, "make_oracle_golden.py"))
    mk = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mk)
    w, r, dense = mk.compute()
    ref = _load("oracle_tiny_fp32.json")
    assert r["idx"].tolist() == ref["idx"]
    np.testing.assert_allclose(r["out"], np.array(ref["out"]), rtol=0, atol=1e-9)
    np.testing.assert_allclose(dense, np.array(ref["dense_out"]), rtol=0, atol=1e-9)


# ----------------------------------------------------------------------------- top-k agreement
def test_jaccard_closed_forms():
    a = np.array([[1, 2, 3, 4], [0, 1, 2, 3], [5, 6, 7, 8]])
    b = np.array([[3, 4, 5, 6], [0, 1, 2, 3], [1, 2, 3, 4]])
    # |{3,4}| / |{1..6}|, identical sets, disjoint sets
    np.testing.assert_allclose(oracle.topk_jaccard(a, b), [2 / 6, 1.0, 0.0], rtol=0, atol=1e-15)


def test_jaccard_brute_force():
    rng = np.random.default_rng(3)
    for _ in range(50):
        S, k = int(rng.integers(1, 40)), 0
        k = int(rng.integers(1, S + 1))
        a = np.sort(rng.choice(S, k, replace=False))
        b = np.sort(rng.choice(S, k, replace=False))
        inter = sum(1 for x in a if x in b)
        union = len(np.union1d(a, b))
        assert oracle.topk_jaccard(a[None], b[None])[0] == inter / union
        assert inter / union == inter / (2 * k - inter)


def test_exact_topk_is_the_full_dimension_selection():
    # d = D ranks on q_hat . k_hat = q . k (P orthonormal): the exact top-k
    rng = np.random.default_rng(4)
    B, Hkv, G, D, S, k = 1, 2, 2, 16, 50, 9
    X = rng.standard_normal((256, D))
    P, _ = oracle.pca_basis(X)
    keys = rng.standard_normal((B, Hkv, S, D))
    q = rng.standard_normal((B, Hkv * G, D))
    K_hat = oracle.rotate_keys(keys, np.stack([P, P]), "f64")
    ref = oracle.loki_decode(q, K_hat, np.zeros_like(K_hat), np.stack([P, P]), S, D, k)
    for g in range(Hkv):
        s = sum(keys[0, g] @ q[0, h] for h in range(g * G, (g + 1) * G))
        exact = np.sort(np.argsort(-s, kind="stable")[:k])
        assert oracle.topk_jaccard(ref["idx"][0, g][None], exact[None])[0] == 1.0
