"""Pins for the CPU oracle: every function is checked against something other than itself.

T1 absorbed == unabsorbed; T2 brute-force top-r; T3 equivalence with plain (partial-)RoPE
MHA written with loops; T4 Eckart-Young; T6 softmax edge cases; T7 RoPE relative
property; T8 int4 bounds and hand-derived codes; T9 cache accounting vs printed figures;
T10 fixed pair sets; T11 residual window; T12 2-bit codes; T13 many queries per sequence
as rows of causal self-attention; plus hand-derived fixtures under tests/golden/.
"""

import itertools
import json
import os

import numpy as np
import pytest

import oracle as O
from workloads import PARITY_WORKLOADS, WORKLOADS, generate as gen


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _rand_layer(rng, d, H, n_kv, dh):
    W_q = rng.standard_normal((d, H * dh)) / np.sqrt(d)
    W_k = rng.standard_normal((d, n_kv * dh)) / np.sqrt(d)
    W_v = rng.standard_normal((d, n_kv * dh)) / np.sqrt(d)
    return W_q, W_k, W_v


def _converted_decode(rng, d, H, n_kv, dh, r, d_c, L, absorbed=False, pair_idx=None, svd="joint"):
    """Run the oracle's convert -> append -> decode on random data; also return raw pieces."""
    W_q, W_k, W_v = _rand_layer(rng, d, H, n_kv, dh)
    if pair_idx is None:
        q_cal = rng.standard_normal((64, d)) @ W_q
        k_cal = rng.standard_normal((64, d)) @ W_k
        contrib = O.pair_scores(q_cal.reshape(64, H, dh), k_cal.reshape(64, n_kv, dh))
        pair_idx = O.select_pairs(contrib, r)
    low_rank = O.svd_split if svd == "split" else O.svd_joint
    W_dkv, W_uk, W_uv, _ = low_rank(W_k, W_v, pair_idx, d_c, dh)
    W_kr = O.krope_weights(W_k, pair_idx, dh)
    theta = O.rope_theta(dh, 10000.0)
    x = rng.standard_normal((L, d))
    c, kr = O.append(x, np.arange(L), W_dkv, W_kr, pair_idx, theta)
    q = (rng.standard_normal(d) @ W_q).reshape(H, dh)
    f = O.decode_absorbed if absorbed else O.decode_unabsorbed
    o = f(q, c, kr, W_uk, W_uv, pair_idx, theta)
    k = (x @ W_k).reshape(L, n_kv, dh)
    v = (x @ W_v).reshape(L, n_kv, dh)
    return o, q, k, v, theta, pair_idx, (c, kr, W_uk, W_uv)


# ------------------------------------------------------------------ fixtures
def test_pair_scores_worked_examples(golden_dir):
    fx = _load(golden_dir, "pair_score_worked.json")
    for case in fx["cases"]:
        q = np.asarray(case["q_cal"], dtype=np.float64)
        k = np.asarray(case["k_cal"], dtype=np.float64)
        contrib = O.pair_scores(q, k)
        np.testing.assert_allclose(contrib, case["contrib"], rtol=0, atol=1e-12)
        assert O.select_pairs(contrib, case["r"]).tolist() == case["pair_idx"]


def test_rope_worked_examples(golden_dir):
    fx = _load(golden_dir, "rope_worked.json")
    theta = O.rope_theta(fx["head_dim"], fx["base"])
    np.testing.assert_allclose(theta, fx["theta"], rtol=1e-15)
    for case in fx["cases"]:
        v = np.asarray(case["vector"], dtype=np.float64).reshape(-1, 2)
        out = O.rotate(v, case["pos"], theta).reshape(-1)
        np.testing.assert_allclose(out, case["expected"], rtol=0, atol=1e-15)


def test_int4_worked_examples(golden_dir):
    fx = _load(golden_dir, "int4_worked.json")
    for case in fx["cases"]:
        c = np.asarray(case["values"], dtype=np.float64)[None]
        codes, scales = O.quant_int4_g32(c)
        assert float(scales[0, 0]) == case["scale"], case["name"]
        assert codes[0].tolist() == case["codes"], case["name"]
    pk = fx["packing"]
    packed = O.pack_int4(np.asarray(pk["codes"], dtype=np.int8)[None])
    assert packed[0].tolist() == pk["bytes"]
    assert O.unpack_int4(packed)[0].tolist() == pk["codes"]


# ------------------------------------------------------------------ T1 / T3
@pytest.mark.parametrize("H,n_kv", [(4, 4), (6, 2)])
def test_T1_absorbed_equals_unabsorbed(H, n_kv):
    rng = np.random.default_rng(11)
    a = _converted_decode(rng, 48, H, n_kv, 16, 3, 20, 37)
    rng = np.random.default_rng(11)
    b = _converted_decode(rng, 48, H, n_kv, 16, 3, 20, 37, absorbed=True)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("H,n_kv", [(4, 4), (6, 3)])
def test_T3_all_pairs_full_rank_is_rope_mha(H, n_kv):
    """r = d_h/2 and d_c = rank: the converted layer reproduces the original RoPE MHA."""
    rng = np.random.default_rng(5)
    dh, d, L = 8, 64, 13
    pair_idx = np.tile(np.arange(dh // 2), (n_kv, 1))
    d_c = n_kv * dh  # W_kv = W_v only (no NoPE key dims): rank n_kv*d_h
    o, q, k, v, theta, _, _ = _converted_decode(rng, d, H, n_kv, dh, dh // 2, d_c, L, pair_idx=pair_idx)
    ref = O.mha_textbook_rope(q, k, v, theta)
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-11)


def test_T3_no_rope_full_rank_is_nope_mha():
    rng = np.random.default_rng(6)
    H, n_kv, dh, d, L = 4, 2, 8, 64, 9
    pair_idx = np.zeros((n_kv, 0), dtype=np.int64)
    o, q, k, v, theta, _, _ = _converted_decode(rng, d, H, n_kv, dh, 0, 2 * n_kv * dh, L, pair_idx=pair_idx)
    ref = O.mha_textbook_rope(q, k, v, theta, rope_pairs=[[] for _ in range(n_kv)])
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("H,n_kv", [(4, 4), (8, 2)])
def test_T3_partial_rope_full_rank_matches_masked_rope_mha(H, n_kv):
    """Any kept-pair set with a full-rank latent equals MHA with RoPE on exactly those pairs."""
    rng = np.random.default_rng(7)
    dh, d, L, r = 8, 96, 11, 2
    d_c = n_kv * (dh - 2 * r) + n_kv * dh
    o, q, k, v, theta, pair_idx, _ = _converted_decode(rng, d, H, n_kv, dh, r, d_c, L)
    ref = O.mha_textbook_rope(q, k, v, theta, rope_pairs=pair_idx)
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-11)


# ------------------------------------------------------------------ T2
def test_T2_topr_maximises_total_score_brute_force():
    rng = np.random.default_rng(3)
    for trial in range(20):
        T, H, n_kv, dh, r = 5, 4, 2, 12, 3
        q = rng.standard_normal((T, H, dh)) * rng.lognormal(0, 0.7, size=(1, H, dh))
        k = rng.standard_normal((T, n_kv, dh)) * rng.lognormal(0, 0.7, size=(1, n_kv, dh))
        contrib = O.pair_scores(q, k)
        sel = O.select_pairs(contrib, r)
        for g in range(n_kv):
            best = max(itertools.combinations(range(dh // 2), r),
                       key=lambda s: (sum(contrib[g, list(s)]), [-x for x in s]))
            assert tuple(sel[g]) == tuple(sorted(best))


def test_T2_score_is_attained_cauchy_schwarz_bound():
    """Per token, ||q_pair||*||k_pair|| is the max over relative rotation of |q_pair . R k_pair|."""
    rng = np.random.default_rng(4)
    T, H, n_kv, dh = 3, 2, 1, 6
    q = rng.standard_normal((T, H, dh))
    k = rng.standard_normal((T, n_kv, dh))
    phis = np.linspace(0, 2 * np.pi, 200001)
    brute = np.zeros((n_kv, dh // 2))
    for t in range(T):
        for h in range(H):
            for kk in range(dh // 2):
                a = q[t, h, 2 * kk:2 * kk + 2]
                b = k[t, 0, 2 * kk:2 * kk + 2]
                rb0 = b[0] * np.cos(phis) - b[1] * np.sin(phis)
                rb1 = b[0] * np.sin(phis) + b[1] * np.cos(phis)
                brute[0, kk] += np.max(np.abs(a[0] * rb0 + a[1] * rb1)) / (T * H)
    np.testing.assert_allclose(O.pair_scores(q, k), brute, rtol=1e-8)


# ------------------------------------------------------------------ T4
def test_T4_eckart_young_and_orthonormal_down_projection():
    rng = np.random.default_rng(8)
    d, n_kv, dh, r, d_c = 80, 3, 16, 2, 24
    _, W_k, W_v = _rand_layer(rng, d, 3, n_kv, dh)
    pair_idx = np.array([[0, 5], [1, 7], [2, 3]])
    W_dkv, W_uk, W_uv, s = O.svd_joint(W_k, W_v, pair_idx, d_c, dh)
    np.testing.assert_allclose(W_dkv.T @ W_dkv, np.eye(d_c), atol=1e-12)
    _, nope = O.split_dims(pair_idx, dh)
    W_kv = np.concatenate([W_k[:, g * dh + nope[g]] for g in range(n_kv)] + [W_v], axis=1)
    recon = np.concatenate([W_dkv @ W_uk[g] for g in range(n_kv)] + [W_dkv @ W_uv[g] for g in range(n_kv)], axis=1)
    err = np.linalg.norm(W_kv - recon) ** 2
    np.testing.assert_allclose(err, np.sum(s[d_c:] ** 2), rtol=1e-9)
    # the split keeps per-head blocks in place: head g's NoPE key columns come from W_uk[g]
    assert W_uk.shape == (n_kv, d_c, dh - 2 * r) and W_uv.shape == (n_kv, d_c, dh)


def test_split_dims_and_krope_columns():
    pair_idx = np.array([[1, 3]])
    rope, nope = O.split_dims(pair_idx, 8)
    assert rope.tolist() == [[2, 3, 6, 7]] and nope.tolist() == [[0, 1, 4, 5]]
    W_k = np.arange(3 * 8, dtype=np.float64).reshape(3, 8)
    assert O.krope_weights(W_k, pair_idx, 8)[:, 0, :].tolist() == W_k[:, [2, 3, 6, 7]].tolist()


# ------------------------------------------------------------------ T6
def _tiny_conv(rng, d=40, H=4, n_kv=2, dh=8, r=1, d_c=12):
    W_q, W_k, W_v = _rand_layer(rng, d, H, n_kv, dh)
    pair_idx = np.array([[0], [2]])
    W_dkv, W_uk, W_uv, _ = O.svd_joint(W_k, W_v, pair_idx, d_c, dh)
    W_kr = O.krope_weights(W_k, pair_idx, dh)
    return W_q, W_dkv, W_kr, W_uk, W_uv, pair_idx, O.rope_theta(dh, 10000.0)


def test_T6_softmax_edge_cases():
    rng = np.random.default_rng(9)
    W_q, W_dkv, W_kr, W_uk, W_uv, pair_idx, theta = _tiny_conv(rng)
    H, G = 4, 2
    # L = 1: output is V of the only token
    x = rng.standard_normal((1, 40))
    c, kr = O.append(x, np.arange(1), W_dkv, W_kr, pair_idx, theta)
    q = (rng.standard_normal(40) @ W_q).reshape(H, 8)
    o = O.decode_unabsorbed(q, c, kr, W_uk, W_uv, pair_idx, theta)
    for h in range(H):
        np.testing.assert_allclose(o[h], c[0] @ W_uv[h // G], rtol=1e-12, atol=1e-13)
    # q = 0: uniform weights, output is the mean of V
    x = rng.standard_normal((7, 40))
    c, kr = O.append(x, np.arange(7), W_dkv, W_kr, pair_idx, theta)
    o = O.decode_unabsorbed(np.zeros((H, 8)), c, kr, W_uk, W_uv, pair_idx, theta)
    for h in range(H):
        np.testing.assert_allclose(o[h], (c @ W_uv[h // G]).mean(axis=0), rtol=1e-12, atol=1e-13)
    # identical latent and no RoPE score difference (kr = 0): output equals that V
    c = np.tile(c[:1], (5, 1))
    kr = np.zeros((5, 2, 2))
    o = O.decode_unabsorbed(q, c, kr, W_uk, W_uv, pair_idx, theta)
    for h in range(H):
        np.testing.assert_allclose(o[h], c[0] @ W_uv[h // G], rtol=1e-12, atol=1e-13)


def test_T6s_softmax_scale():
    """A caller-chosen score scale (the boundary's softmax_scale): the default is the
    original layer's 1/sqrt(d_h); the scores are linear in q (the rotation is linear), so
    scale k/sqrt(d_h) equals the default decode of k*q; scale 0 gives uniform weights."""
    rng = np.random.default_rng(19)
    W_q, W_dkv, W_kr, W_uk, W_uv, pair_idx, theta = _tiny_conv(rng)
    H, G, dh = 4, 2, 8
    x = rng.standard_normal((9, 40))
    c, kr = O.append(x, np.arange(9), W_dkv, W_kr, pair_idx, theta)
    q = (rng.standard_normal(40) @ W_q).reshape(H, dh)
    base = O.decode_unabsorbed(q, c, kr, W_uk, W_uv, pair_idx, theta)
    np.testing.assert_array_equal(O.decode_unabsorbed(q, c, kr, W_uk, W_uv, pair_idx, theta,
                                                      scale=1.0 / np.sqrt(dh)), base)
    for k in (0.37, 2.5):
        np.testing.assert_allclose(O.decode_unabsorbed(q, c, kr, W_uk, W_uv, pair_idx, theta, scale=k / np.sqrt(dh)),
                                   O.decode_unabsorbed(k * q, c, kr, W_uk, W_uv, pair_idx, theta),
                                   rtol=1e-12, atol=1e-13)
    assert not np.allclose(O.decode_unabsorbed(q, c, kr, W_uk, W_uv, pair_idx, theta, scale=2.5 / np.sqrt(dh)), base)
    o0 = O.decode_unabsorbed(q, c, kr, W_uk, W_uv, pair_idx, theta, scale=0.0)
    for h in range(H):
        np.testing.assert_allclose(o0[h], (c @ W_uv[h // G]).mean(axis=0), rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ T7
def test_T7_rope_relative_position_and_norms():
    rng = np.random.default_rng(10)
    theta = O.rope_theta(16, 10000.0)
    q = rng.standard_normal((8, 2))
    k = rng.standard_normal((8, 2))
    for p, t, delta in [(5, 2, 17), (100, 99, 1000), (0, 0, 12345)]:
        s0 = np.sum(O.rotate(q, p, theta) * O.rotate(k, t, theta))
        s1 = np.sum(O.rotate(q, p + delta, theta) * O.rotate(k, t + delta, theta))
        assert abs(s0 - s1) < 1e-10
    r = O.rotate(q, 37, theta)
    np.testing.assert_allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-14)
    np.testing.assert_array_equal(O.rotate(q, 0, theta), q)


def test_T7_append_rotates_each_kept_pair_at_its_own_frequency():
    rng = np.random.default_rng(12)
    d, dh = 16, 8
    W_dkv = rng.standard_normal((d, 4))
    pair_idx = np.array([[1, 3]])
    W_kr = rng.standard_normal((d, 1, 4))
    theta = O.rope_theta(dh, 10000.0)
    x = rng.standard_normal((3, d))
    c, kr = O.append(x, np.array([0, 5, 9]), W_dkv, W_kr, pair_idx, theta)
    raw = np.einsum("nd,dj->nj", x, W_kr[:, 0, :])
    for n, p in enumerate([0, 5, 9]):
        for j, kk in enumerate([1, 3]):
            a, b = raw[n, 2 * j], raw[n, 2 * j + 1]
            ang = p * theta[kk]
            assert abs(kr[n, 0, 2 * j] - (a * np.cos(ang) - b * np.sin(ang))) < 1e-12
            assert abs(kr[n, 0, 2 * j + 1] - (a * np.sin(ang) + b * np.cos(ang))) < 1e-12
    np.testing.assert_allclose(c, x @ W_dkv, rtol=1e-14)


# ------------------------------------------------------------------ T8
def test_T8_int4_error_bound_and_round_trip():
    rng = np.random.default_rng(13)
    c = rng.standard_normal((50, 128)) * rng.lognormal(0, 1, size=(50, 1))
    codes, scales = O.quant_int4_g32(c)
    assert codes.min() >= -7 and codes.max() <= 7
    deq = O.dequant_int4_g32(codes, scales)
    sc = np.repeat(scales.astype(np.float64), 32, axis=1)
    c32 = c.astype(np.float32).astype(np.float64)
    # within half a step (plus the float32 division's rounding), and the group max lands on +-7
    assert np.all(np.abs(deq - c32) <= sc * (0.5 + 1e-6) + 1e-30)
    assert np.all(np.abs(codes.reshape(50, 4, 32)).max(axis=-1) == 7)
    # exactly representable values round-trip exactly
    codes2, scales2 = O.quant_int4_g32(deq)
    np.testing.assert_array_equal(codes2, codes)
    np.testing.assert_array_equal(scales2, scales)
    np.testing.assert_array_equal(O.unpack_int4(O.pack_int4(codes)), codes)


# ------------------------------------------------------------------ T9
def test_T9_cache_accounting_matches_printed_reductions(golden_dir):
    fx = _load(golden_dir, "cache_reduction.json")
    m = fx["llama2_7b"]
    mha = O.mha_cache_bytes_per_token(m["n_heads"], m["head_dim"], m["elem_bytes"])
    assert mha == 16384
    for row in fx["rows"]:
        if "gqa_kv_heads" in row:
            got = 1 - O.mha_cache_bytes_per_token(row["gqa_kv_heads"], m["head_dim"], 2) / mha
        else:
            got = 1 - O.cache_bytes_per_token(row["n_kv"], row["r"], row["d_c"], 2, int4=row["int4"],
                                              count_scales=row.get("count_scales", True)) / mha
        # printed to two decimals (96.875 is printed truncated as 96.87)
        assert abs(100 * got - row["printed_percent"]) < 0.01, row["name"]


def test_T9_workload_cache_bytes():
    per_tok = {w.name: O.cache_bytes_per_token(w.n_kv_heads, w.r_pairs, w.d_c,
                                               4 if w.dtype == "f32" else 2, int4=w.cache == "int4_g32")
               for w in WORKLOADS}
    assert per_tok["tiny_f32"] == 192 and per_tok["smollm135m_gqa_bf16"] == 112
    assert per_tok["llama2_7b_bf16"] == 1024 and per_tok["llama2_7b_ragged_bf16"] == 640
    assert per_tok["llama2_7b_int4"] == 584


# ------------------------------------------------------------------ generators
def test_generators_are_seeded_and_cast():
    wl = PARITY_WORKLOADS[2]
    a = gen.layer_weights(wl)
    b = gen.layer_weights(wl)
    np.testing.assert_array_equal(a["W_q"], b["W_q"])
    # bf16 values: at most 8 significant bits
    v = a["W_k"].ravel()[:1000]
    np.testing.assert_array_equal(gen.cast(v, "bf16"), v)
    x0 = gen.context_tokens(wl, 1, 50)
    x1 = gen.context_tokens(wl, 1, 80)[:50]
    np.testing.assert_array_equal(x0, x1)
    assert gen.seq_lens(WORKLOADS[3]).min() >= 1024 and gen.seq_lens(WORKLOADS[3]).max() <= 32768


# ------------------------------------------------------------------ T10 fixed pair sets
def test_T10_fixed_pair_sets_hand_written():
    """README §Fine-Tuning (partial-RoPE versions) / Notes §消融实验: the high, low,
    uniform and full strategies, written out by hand for small cases."""
    assert O.fixed_pairs("high", 128, 4, 1).tolist() == [[0, 1, 2, 3]]
    assert O.fixed_pairs("low", 128, 4, 1).tolist() == [[60, 61, 62, 63]]
    assert O.fixed_pairs("uniform", 128, 4, 1).tolist() == [[0, 16, 32, 48]]
    assert O.fixed_pairs("uniform", 12, 4, 1).tolist() == [[0, 1, 3, 4]]   # P = 6: 0, 1.5, 3, 4.5
    assert O.fixed_pairs("full", 8, 4, 2).tolist() == [[0, 1, 2, 3], [0, 1, 2, 3]]
    with pytest.raises(ValueError):
        O.fixed_pairs("full", 8, 3, 1)


@pytest.mark.parametrize("dh,r", [(32, 2), (64, 4), (128, 4), (128, 13), (64, 31)])
def test_T10_fixed_pairs_frequency_meaning(dh, r):
    """'high' keeps the fastest-rotating pairs, 'low' the slowest (theta_k from rope_theta,
    pair 0 fastest); 'uniform' starts at pair 0 with steps of floor or ceil of P/r."""
    theta = O.rope_theta(dh, 10000.0)
    P = dh // 2
    for strat, faster in (("high", True), ("low", False)):
        ks = O.fixed_pairs(strat, dh, r, 1)[0]
        rest = [k for k in range(P) if k not in set(ks.tolist())]
        if rest:
            if faster:
                assert theta[ks].min() > theta[rest].max()
            else:
                assert theta[ks].max() < theta[rest].min()
    u = O.fixed_pairs("uniform", dh, r, 1)[0]
    assert u[0] == 0 and len(set(u.tolist())) == r and u.max() < P
    steps = np.diff(u)
    assert set(steps.tolist()) <= {P // r, -(-P // r)}


def test_T10_full_strategy_is_every_pair_and_rope_mha():
    """Full RoPE keeps every pair, the same set the 2-norm top-P selection returns; at
    full latent rank the converted layer then reproduces textbook RoPE MHA (pin T3)."""
    wl = WORKLOADS[0].with_(name="tiny_full_rope", r_pairs=WORKLOADS[0].head_dim // 2,
                            d_c=WORKLOADS[0].n_kv_heads * (2 * WORKLOADS[0].head_dim))
    full = O.fixed_pairs("full", wl.head_dim, wl.r_pairs, wl.n_kv_heads)
    contrib = np.random.default_rng(7).random((wl.n_kv_heads, wl.head_dim // 2))
    assert np.array_equal(full, O.select_pairs(contrib, wl.r_pairs))


# ------------------------------------------------------------------ T4s SVD_split
def test_T4s_split_eckart_young_per_part_and_zero_blocks():
    """SVD_split: each half is the truncated SVD of its own matrix (Eckart-Young per part,
    orthonormal columns per half); the key up-projection reads only c_k and the value
    up-projection only c_v."""
    rng = np.random.default_rng(18)
    d, n_kv, dh, r, d_c = 80, 3, 16, 2, 24
    _, W_k, W_v = _rand_layer(rng, d, 3, n_kv, dh)
    pair_idx = np.array([[0, 5], [1, 7], [2, 3]])
    W_dkv, W_uk, W_uv, (s_k, s_v) = O.svd_split(W_k, W_v, pair_idx, d_c, dh)
    dk = d_c // 2
    U_k, U_v = W_dkv[:, :dk], W_dkv[:, dk:]
    np.testing.assert_allclose(U_k.T @ U_k, np.eye(dk), atol=1e-12)
    np.testing.assert_allclose(U_v.T @ U_v, np.eye(d_c - dk), atol=1e-12)
    assert np.all(W_uk[:, dk:] == 0) and np.all(W_uv[:, :dk] == 0)
    _, nope = O.split_dims(pair_idx, dh)
    Wk_nope = np.concatenate([W_k[:, g * dh + nope[g]] for g in range(n_kv)], axis=1)
    rec_k = np.concatenate([W_dkv @ W_uk[g] for g in range(n_kv)], axis=1)
    rec_v = np.concatenate([W_dkv @ W_uv[g] for g in range(n_kv)], axis=1)
    np.testing.assert_allclose(np.linalg.norm(Wk_nope - rec_k) ** 2, np.sum(s_k[dk:] ** 2), rtol=1e-9)
    np.testing.assert_allclose(np.linalg.norm(W_v - rec_v) ** 2, np.sum(s_v[d_c - dk:] ** 2), rtol=1e-9)
    # at the same total rank the joint SVD of the concatenation loses no more energy
    _, _, _, s_j = O.svd_joint(W_k, W_v, pair_idx, d_c, dh)
    assert np.sum(s_k[dk:] ** 2) + np.sum(s_v[d_c - dk:] ** 2) >= np.sum(s_j[d_c:] ** 2) - 1e-9


@pytest.mark.parametrize("H,n_kv", [(4, 4), (8, 2)])
def test_T3s_split_full_rank_matches_masked_rope_mha(H, n_kv):
    """SVD_split with each half at full rank reproduces MHA with RoPE on the kept pairs."""
    rng = np.random.default_rng(19)
    dh, d, L, r = 8, 96, 11, 2
    d_c = 2 * max(n_kv * (dh - 2 * r), n_kv * dh)
    o, q, k, v, theta, pair_idx, _ = _converted_decode(rng, d, H, n_kv, dh, r, d_c, L, svd="split")
    ref = O.mha_textbook_rope(q, k, v, theta, rope_pairs=pair_idx)
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-11)


# ------------------------------------------------------------------ T11 residual window
def test_T11_residual_window_special_cases_and_rows():
    rng = np.random.default_rng(23)
    L, dc = 5, 64
    c = rng.standard_normal((L, dc))
    codes, scales = O.quant_int4_g32(c)
    deq = O.dequant_int4_g32(codes, scales)
    plain = gen.cast(c, "bf16")
    np.testing.assert_array_equal(O.residual_window(deq, plain, 0), deq)        # no window: int4 only
    np.testing.assert_array_equal(O.residual_window(deq, plain, L), plain)      # window covers all
    np.testing.assert_array_equal(O.residual_window(deq, plain, 128), plain)
    got = O.residual_window(deq, plain, 2)                                       # rows 3, 4 are recent
    for t, src in enumerate([deq, deq, deq, plain, plain]):
        np.testing.assert_array_equal(got[t], src[t])


def test_T11_ring_with_position_tags_selects_the_window():
    """A ring of W slots (slot t % W, each slot keeping the largest position written to it,
    whatever the order inside one append call), read for t >= L - W when the slot's tag is
    t, selects exactly the rows residual_window takes from the unquantised values."""
    rng = np.random.default_rng(29)
    W = 8
    for trial in range(200):
        L = int(rng.integers(0, 40))
        tags = np.full(W, -1)
        done = 0
        while done < L:          # in-order calls of random size; tokens of a call in random order
            n = int(rng.integers(1, 20))
            call = rng.permutation(np.arange(done, min(L, done + n)))
            for t in call:
                tags[t % W] = max(tags[t % W], t)
            done = min(L, done + n)
        from_ring = np.array([t >= L - W and tags[t % W] == t for t in range(L)], dtype=bool)
        quant = np.zeros((L, 1))
        plain = np.ones((L, 1))
        sel = O.residual_window(quant, plain, W)[:, 0] == 1
        np.testing.assert_array_equal(from_ring, sel)


def test_T11_decode_over_window_reduces_to_pinned_decodes():
    """Window >= L: the decode over the plain (bf16) latents; window 0: over the int4 values."""
    rng = np.random.default_rng(31)
    o, q, k, v, theta, pair_idx, (c, kr, W_uk, W_uv) = _converted_decode(rng, 64, 4, 2, 16, 2, 32, 40)
    codes, scales = O.quant_int4_g32(c)
    deq = O.dequant_int4_g32(codes, scales)
    plain = gen.cast(c, "bf16")
    dec = lambda cc: O.decode_unabsorbed(q, cc, kr, W_uk, W_uv, pair_idx, theta)  # noqa: E731
    np.testing.assert_array_equal(dec(O.residual_window(deq, plain, 40)), dec(plain))
    np.testing.assert_array_equal(dec(O.residual_window(deq, plain, 0)), dec(deq))
    mixed = dec(O.residual_window(deq, plain, 16))
    assert not np.array_equal(mixed, dec(deq)) and not np.array_equal(mixed, dec(plain))


# ------------------------------------------------------------------ T12 2-bit latent
def test_T12_int2_hand_derived_codes_and_bytes():
    g = np.zeros((1, 32))
    g[0, :8] = [3.0, -3.0, 1.4, -1.6, 1.5, -1.5, 0.2, 2.9]
    codes, scales = O.quant_int2_g32(g)
    assert scales[0, 0] == np.float16(3.0)
    # c/s = 1, -1, 0.467, -0.533, 0.5 (half to even: 0), -0.5 (0), 0.067, 0.967
    assert codes[0, :8].tolist() == [1, -1, 0, -1, 0, 0, 0, 1]
    assert np.all(codes[0, 8:] == 0)
    # bytes: element 4i + k in bits 2k..2k+1, two's complement (-1 = 0b11)
    packed = O.pack_int2(codes)
    assert packed[0, 0] == (1 | (3 << 2) | (0 << 4) | (3 << 6))
    assert packed[0, 1] == (0 | (0 << 2) | (0 << 4) | (1 << 6))
    np.testing.assert_array_equal(O.unpack_int2(packed), codes)
    # every 2-bit field value, two's complement: 00 -> 0, 01 -> 1, 11 -> -1, 10 -> -2
    byte = np.array([[0b10_11_01_00]], dtype=np.uint8)
    assert O.unpack_int2(byte)[0].tolist() == [0, 1, -1, -2]
    z, zs = O.quant_int2_g32(np.zeros((2, 64)))
    assert np.all(z == 0) and np.all(zs == 0)


def test_T12_int2_error_bound_and_round_trip():
    rng = np.random.default_rng(37)
    c = rng.standard_normal((40, 128)) * rng.lognormal(0, 1, size=(40, 1))
    codes, scales = O.quant_int2_g32(c)
    assert set(np.unique(codes).tolist()) <= {-1, 0, 1}
    deq = O.dequant_int2_g32(codes, scales)
    sc = np.repeat(scales.astype(np.float64), 32, axis=1)
    c32 = c.astype(np.float32).astype(np.float64)
    # within half a step (plus the fp16 rounding of the scale), and the group max lands on +-1
    assert np.all(np.abs(deq - c32) <= sc * (0.5 + 1e-3) + 1e-30)
    assert np.all(np.abs(codes.reshape(40, 4, 32)).max(axis=-1) == 1)
    codes2, scales2 = O.quant_int2_g32(deq)
    np.testing.assert_array_equal(codes2, codes)
    np.testing.assert_array_equal(scales2, scales)
    np.testing.assert_array_equal(O.unpack_int2(O.pack_int2(codes)), codes)
    # 2 bits lose more than 4 on the same latents
    c4, s4 = O.quant_int4_g32(c)
    assert np.linalg.norm(O.dequant_int4_g32(c4, s4) - c32) < np.linalg.norm(deq - c32)


# ------------------------------------------------------------------ T13 many queries per sequence
def _causal_rope_mha(x, W_q, W_k, W_v, H, n_kv, dh, pair_idx, theta):
    """Causal self-attention of the original layer over a whole sequence as one masked score
    matrix: token i's query (rotated at i on the kept pairs of its KV head) against every key
    j <= i (rotated at j), scale 1/sqrt(d_h).  Returns o [L][H][d_h]."""
    L = x.shape[0]
    G = H // n_kv
    q = (x @ W_q).reshape(L, H, dh)
    k = (x @ W_k).reshape(L, n_kv, dh)
    v = (x @ W_v).reshape(L, n_kv, dh)
    pos = np.arange(L, dtype=np.float64)
    o = np.zeros((L, H, dh))
    for h in range(H):
        g = h // G
        qh, kg = q[:, h].copy(), k[:, g].copy()
        for kk in pair_idx[g]:
            ang = pos * theta[kk]
            cos, sin = np.cos(ang), np.sin(ang)
            for m in (qh, kg):
                a, b = m[:, 2 * kk].copy(), m[:, 2 * kk + 1].copy()
                m[:, 2 * kk], m[:, 2 * kk + 1] = a * cos - b * sin, a * sin + b * cos
        s = qh @ kg.T / np.sqrt(dh)
        s[np.triu_indices(L, 1)] = -np.inf          # key j > query i: masked
        p = np.exp(s - s.max(axis=1, keepdims=True))
        o[:, h] = (p / p.sum(axis=1, keepdims=True)) @ v[:, g]
    return o


@pytest.mark.parametrize("H,n_kv", [(4, 4), (6, 3)])
def test_T13_chunk_queries_are_rows_of_causal_attention(H, n_kv):
    """A chunk of the newest Q tokens, each query decoded over its own prefix [0, L-Q+i] and
    rotated at L-Q+i (the reading the chunk kernel's parity tests use), equals the last Q rows
    of the original layer's causal self-attention when the latent has full rank."""
    rng = np.random.default_rng(41)
    dh, d, L, r, Q = 8, 96, 23, 2, 7
    W_q, W_k, W_v = _rand_layer(rng, d, H, n_kv, dh)
    pair_idx = np.stack([np.sort(rng.choice(dh // 2, r, replace=False)) for _ in range(n_kv)])
    d_c = n_kv * (dh - 2 * r) + n_kv * dh
    W_dkv, W_uk, W_uv, _ = O.svd_joint(W_k, W_v, pair_idx, d_c, dh)
    theta = O.rope_theta(dh, 10000.0)
    x = rng.standard_normal((L, d))
    c, kr = O.append(x, np.arange(L), W_dkv, O.krope_weights(W_k, pair_idx, dh), pair_idx, theta)
    ref = _causal_rope_mha(x, W_q, W_k, W_v, H, n_kv, dh, pair_idx, theta)
    q = (x @ W_q).reshape(L, H, dh)
    for i in range(Q):
        p = L - Q + i
        got = O.decode_unabsorbed(q[p], c[:p + 1], kr[:p + 1], W_uk, W_uv, pair_idx, theta)
        np.testing.assert_allclose(got, ref[p], rtol=1e-10, atol=1e-11)
    # the prefix is inclusive: leaving out the query's own token changes the result
    p = L - 1
    short = O.decode_unabsorbed(q[p], c[:p], kr[:p], W_uk, W_uv, pair_idx, theta)
    assert np.abs(short - ref[p]).max() > 1e-3
