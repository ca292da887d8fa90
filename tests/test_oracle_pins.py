"""Pins of the fp64 CPU oracle against what the pages and mathematics fix.

Each test names the passage it follows.  Page shorthand used below:
  HEADS  = xuesongtap "attention-head" article
  MHAVS  = astro-blog "MHA vs MQA vs GQA vs MLA" article
  EVOL   = toolsku "AI演算法注意力機制演進" article
  LESSON = llmdeepdive lesson "MQA, GQA e MLA"
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle as orc
from workloads import BLOCK_SIZE, make_block_table

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _paged_from_dense(K, V, block_size=BLOCK_SIZE, perm_seed=None):
    """Lay dense per-sequence caches [B][H_kv][T][d] into the paged format.

    Returns (k_cache, v_cache, block_table).  With perm_seed, the physical
    blocks are a random permutation; otherwise the identity.
    """
    B, H, T, d = K.shape
    nb = (T + block_size - 1) // block_size
    total = B * nb
    ids = (np.random.default_rng(perm_seed).permutation(total)
           if perm_seed is not None else np.arange(total))
    kc = np.zeros((total, H, block_size, d), dtype=K.dtype)
    vc = np.zeros_like(kc)
    table = np.full((B, nb), -1, dtype=np.int32)
    for b in range(B):
        for i in range(nb):
            phys = ids[b * nb + i]
            table[b, i] = phys
            n = min(block_size, T - i * block_size)
            kc[phys, :, :n] = K[b, :, i * block_size:i * block_size + n]
            vc[phys, :, :n] = V[b, :, i * block_size:i * block_size + n]
    return kc, vc, table


# ---------------------------------------------------------------- worked case
def test_hand_computable_mha_case():
    """MHAVS "small-matrix" MHA example setup (d_k=2, h=2, seq_len=4, 4x2
    matrices; its numbers did not survive extraction), with a substitute whose
    softmax has a closed form: keys e1, e2, e1+e2, 0."""
    K = np.array([[1, 0], [0, 1], [1, 1], [0, 0]], dtype=np.float64)
    V = np.array([[1, 2], [3, -1], [-2, 5], [7, 0]], dtype=np.float64)
    q = np.array([[[1.0, 0.0], [0.0, 1.0]]])          # B=1, two heads
    # head 0 uses K, V; head 1 uses its own (here: rows permuted) K, V.
    K1 = K[[1, 0, 3, 2]]
    V1 = V[[2, 3, 0, 1]]
    Kd = np.stack([K, K1])[None]                       # [1][2][4][2]
    Vd = np.stack([V, V1])[None]
    kc, vc, table = _paged_from_dense(Kd, Vd, block_size=4)
    scale = 1.0 / math.sqrt(2.0)
    out, probs = orc.decode_gqa(q, kc, vc, np.array([4]), table, scale,
                                return_probs=True)
    e = math.exp(scale)
    a, b = e / (2 * e + 2), 1.0 / (2 * e + 2)
    # head 0: q=e1 -> scores [1,0,1,0]/sqrt2
    p0 = np.array([a, b, a, b])
    # head 1: q=e2 against rows [e2, e1, 0, e1+e2] -> scores [1,0,0,1]/sqrt2
    p1 = np.array([a, b, b, a])
    np.testing.assert_allclose(probs[0, 0], p0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(probs[0, 1], p1, rtol=0, atol=1e-15)
    np.testing.assert_allclose(out[0, 0], p0 @ V, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[0, 1], p1 @ V1, rtol=0, atol=1e-14)


# ----------------------------------------------------- textbook special cases
def _rand_problem(rng, B, H_q, H_kv, T, d, block_size=BLOCK_SIZE):
    q = rng.standard_normal((B, H_q, d))
    K = rng.standard_normal((B, H_kv, T, d))
    V = rng.standard_normal((B, H_kv, T, d))
    return q, K, V


def test_single_token_returns_its_value_row():
    """T=1: softmax over one key is 1, so out = v_0 (HEADS §1 equation)."""
    rng = np.random.default_rng(1)
    q, K, V = _rand_problem(rng, 2, 4, 2, 1, 16)
    kc, vc, table = _paged_from_dense(K, V)
    out = orc.decode_gqa(q, kc, vc, np.array([1, 1]), table, 0.25)
    for b in range(2):
        for h in range(4):
            np.testing.assert_array_equal(out[b, h], V[b, h // 2, 0])


def test_identical_keys_give_mean_of_values():
    """Identical keys -> equal scores -> uniform p -> mean of V (HEADS §1)."""
    rng = np.random.default_rng(2)
    T, d = 70, 8
    K = np.broadcast_to(rng.standard_normal(d), (1, 1, T, d)).copy()
    V = rng.standard_normal((1, 1, T, d))
    q = rng.standard_normal((1, 1, d))
    kc, vc, table = _paged_from_dense(K, V)
    out, probs = orc.decode_gqa(q, kc, vc, np.array([T]), table, 0.3,
                                return_probs=True)
    np.testing.assert_allclose(probs[0, 0], np.full(T, 1.0 / T), atol=1e-16)
    np.testing.assert_allclose(out[0, 0], V[0, 0].mean(axis=0), atol=1e-14)


def test_dominant_score_selects_its_value_row():
    """One score larger than the rest by 40 -> p concentrates on that key."""
    rng = np.random.default_rng(3)
    T, d = 100, 4
    K = np.zeros((1, 1, T, d))
    K[0, 0, 37, 0] = 40.0
    V = rng.standard_normal((1, 1, T, d))
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    kc, vc, table = _paged_from_dense(K, V)
    out = orc.decode_gqa(q, kc, vc, np.array([T]), table, 1.0)
    np.testing.assert_allclose(out[0, 0], V[0, 0, 37], atol=1e-14)


def test_rows_sum_to_one_and_match_library_softmax():
    """Softmax is taken along key positions (HEADS §1): each row of p sums to
    1 and equals scipy's softmax of the scaled dense scores; the output equals
    p @ V computed densely (independent textbook formulation)."""
    rng = np.random.default_rng(4)
    B, H_q, H_kv, T, d = 3, 6, 3, 150, 32
    q, K, V = _rand_problem(rng, B, H_q, H_kv, T, d)
    lens = np.array([150, 1, 97])
    kc, vc, table = _paged_from_dense(K, V, perm_seed=11)
    scale = 1 / math.sqrt(d)
    out, probs = orc.decode_gqa(q, kc, vc, lens, table, scale,
                                return_probs=True)
    G = H_q // H_kv
    for b in range(B):
        for h in range(H_q):
            n = lens[b]
            Kd, Vd = K[b, h // G, :n], V[b, h // G, :n]
            p = scipy.special.softmax(scale * (Kd @ q[b, h]))
            assert abs(probs[b, h, :n].sum() - 1.0) < 1e-14
            np.testing.assert_allclose(probs[b, h, :n], p, rtol=1e-12,
                                       atol=1e-16)
            assert np.all(probs[b, h, n:] == 0)
            np.testing.assert_allclose(out[b, h], p @ Vd, rtol=1e-12,
                                       atol=1e-13)


def test_empty_sequence_gives_zero_row():
    rng = np.random.default_rng(5)
    q, K, V = _rand_problem(rng, 2, 2, 1, 64, 16)
    kc, vc, table = _paged_from_dense(K, V)
    out = orc.decode_gqa(q, kc, vc, np.array([0, 64]), table, 0.25)
    assert np.all(out[0] == 0)
    assert np.any(out[1] != 0)


# ------------------------------------------------------------- head sharing
@pytest.mark.parametrize("case", _golden("head_groups.json")["cases"],
                         ids=lambda c: f"{c['H_q']}q{c['H_kv']}kv")
def test_group_mapping_matches_page(case):
    """HEADS §2 figure and group rule; LESSON (24 over 4 in groups of 6).
    Each KV head gets a distinct constant value row; the output of query head
    h reveals which KV head it read."""
    H_q, H_kv = case["H_q"], case["H_kv"]
    T, d = 5, 4
    K = np.zeros((1, H_kv, T, d))
    V = np.zeros((1, H_kv, T, d))
    for g in range(H_kv):
        V[0, g, :, 0] = g
    q = np.ones((1, H_q, d))
    kc, vc, table = _paged_from_dense(K, V)
    out = orc.decode_gqa(q, kc, vc, np.array([T]), table, 1.0)
    got = [int(round(out[0, h, 0])) for h in range(H_q)]
    assert got == case["kv_head_of_q_head"]


def test_gqa_with_hkv_equal_hq_is_mha_head_by_head():
    """H_kv = H_q is MHA (HEADS §2.2): each head equals a one-head problem."""
    rng = np.random.default_rng(6)
    B, H, T, d = 2, 5, 130, 16
    q, K, V = _rand_problem(rng, B, H, H, T, d)
    kc, vc, table = _paged_from_dense(K, V, perm_seed=3)
    out = orc.decode_gqa(q, kc, vc, np.array([T, 77]), table, 0.25)
    for h in range(H):
        kc1, vc1, t1 = _paged_from_dense(K[:, h:h + 1], V[:, h:h + 1])
        o1 = orc.decode_gqa(q[:, h:h + 1], kc1, vc1, np.array([T, 77]), t1,
                            0.25)
        np.testing.assert_array_equal(out[:, h], o1[:, 0])


@pytest.mark.parametrize("H_q,H_kv", [(8, 1), (24, 4), (32, 8)])
def test_shared_kv_equals_mha_with_replicated_kv(H_q, H_kv):
    """MQA/GQA equal MHA whose K/V are replicated over each group
    (EVOL repeat_kv expansion; HEADS §2.1, §2.2)."""
    rng = np.random.default_rng(7)
    B, T, d = 2, 90, 8
    q, K, V = _rand_problem(rng, B, H_q, H_kv, T, d)
    G = H_q // H_kv
    Krep = np.repeat(K, G, axis=1)
    Vrep = np.repeat(V, G, axis=1)
    kc, vc, t = _paged_from_dense(K, V, perm_seed=5)
    kr, vr, tr = _paged_from_dense(Krep, Vrep, perm_seed=6)
    lens = np.array([T, 41])
    a = orc.decode_gqa(q, kc, vc, lens, t, 0.35)
    b = orc.decode_gqa(q, kr, vr, lens, tr, 0.35)
    np.testing.assert_array_equal(a, b)
    # sensitivity: the wrong (interleaved, h % H_kv) expansion differs
    if H_kv > 1:
        idx = [h % H_kv for h in range(H_q)]
        kw, vw, tw = _paged_from_dense(K[:, idx], V[:, idx])
        c = orc.decode_gqa(q, kw, vw, lens, tw, 0.35)
        assert np.abs(a - c).max() > 1e-3


# ----------------------------------------------------------- sliding window
@pytest.mark.parametrize("case", _golden("window_membership.json")["cases"],
                         ids=lambda c: f"w{c['window']}")
def test_window_membership_matches_page_figure(case):
    """HEADS §3 figure: row i=8, w=3 keeps {6,7,8}; full causal keeps 0..8."""
    T, w = case["T"], case["window"]
    lo, hi = orc.visible_range(T, w)
    assert list(range(lo, hi)) == case["visible"]
    rng = np.random.default_rng(8)
    q, K, V = _rand_problem(rng, 1, 1, 1, T, 4)
    kc, vc, table = _paged_from_dense(K, V)
    _, probs = orc.decode_gqa(q, kc, vc, np.array([T]), table, 0.5, window=w,
                              return_probs=True)
    assert [j for j in range(T) if probs[0, 0, j] > 0] == case["visible"]


def test_window_brute_force_membership():
    """Brute force over small T and w: the visible set is exactly the w most
    recent positions, the current one included (HEADS §3)."""
    for T in range(0, 12):
        for w in range(0, 14):
            lo, hi = orc.visible_range(T, w)
            expect = [j for j in range(T) if w <= 0 or T - 1 - j < w]
            assert list(range(lo, hi)) == expect, (T, w)


def test_window_at_least_T_equals_full_causal():
    """A window w >= T drops nothing: it reduces to full causal attention (HEADS §3)."""
    rng = np.random.default_rng(9)
    q, K, V = _rand_problem(rng, 2, 4, 2, 200, 16)
    kc, vc, table = _paged_from_dense(K, V, perm_seed=1)
    lens = np.array([200, 65])
    full = orc.decode_gqa(q, kc, vc, lens, table, 0.25)
    for w in (200, 201, 10_000):
        np.testing.assert_array_equal(
            orc.decode_gqa(q, kc, vc, lens, table, 0.25, window=w), full)
    part = orc.decode_gqa(q, kc, vc, lens, table, 0.25, window=64)
    assert np.abs(part - full).max() > 1e-3


# ------------------------------------------------------------------- paging
def test_permuted_block_table_equals_identity_table():
    """The block table only relocates blocks: a random permutation gives the
    bit-identical result of the identity layout (paging, Baidu article §4.3)."""
    rng = np.random.default_rng(10)
    q, K, V = _rand_problem(rng, 3, 8, 2, 333, 32)
    lens = np.array([333, 64, 65])
    kc0, vc0, t0 = _paged_from_dense(K, V)
    a = orc.decode_gqa(q, kc0, vc0, lens, t0, 0.2)
    kc, vc, t = _paged_from_dense(K, V, perm_seed=42)
    b = orc.decode_gqa(q, kc, vc, lens, t, 0.2)
    np.testing.assert_array_equal(a, b)


def test_slot_offset_follows_block_table():
    table = np.array([[5, 2, 9], [0, 1, 3]], dtype=np.int32)
    # position 130 of sequence 0 -> logical block 2 -> physical 9, slot 2
    off = orc.slot_offset(table, 0, 130, 64, 4, 3, 16)
    assert off == ((9 * 4 + 3) * 64 + 2) * 16


# --------------------------------------------------------------- precision
def test_bf16_inputs_widen_exactly():
    """bf16 inputs are read as the exact fp64 value of the bf16 number."""
    rng = np.random.default_rng(12)
    qf, Kf, Vf = _rand_problem(rng, 1, 2, 1, 70, 16)
    q16 = torch.from_numpy(qf).to(torch.bfloat16)
    K16 = torch.from_numpy(Kf).to(torch.bfloat16)
    V16 = torch.from_numpy(Vf).to(torch.bfloat16)
    kc, vc, table = _paged_from_dense(K16.double().numpy(),
                                      V16.double().numpy())
    ref = orc.decode_gqa(q16.double().numpy(), kc, vc, np.array([70]), table,
                         0.25)
    kc16 = torch.from_numpy(kc).to(torch.bfloat16)
    vc16 = torch.from_numpy(vc).to(torch.bfloat16)
    got = orc.decode_gqa(q16, kc16, vc16, np.array([70]), table, 0.25)
    np.testing.assert_array_equal(ref, got)


# --------------------------------------------------------------------- MLA
def _mla_problem(rng, B, H, d_c, d_r, d_h, d_v, T):
    latent = rng.standard_normal((B, T, d_c + d_r)) / math.sqrt(d_c + d_r)
    q_c = rng.standard_normal((B, H, d_h))
    q_r = rng.standard_normal((B, H, d_r))
    U_K = rng.standard_normal((H, d_c, d_h)) / math.sqrt(d_c)
    U_V = rng.standard_normal((H, d_c, d_v)) / math.sqrt(d_c)
    return latent, q_c, q_r, U_K, U_V


def _paged_latent(latent, block_size=BLOCK_SIZE, perm_seed=None):
    B, T, w = latent.shape
    K = latent[:, None]                  # treat as one "head"
    kc, _, table = _paged_from_dense(K, K, block_size, perm_seed)
    return kc[:, 0], table


@pytest.mark.parametrize("d_r", [0, 4])
def test_mla_absorbed_equals_explicit(d_r):
    """HEADS §5.2: q^C (U^K)^T c^T = q~ c^T and sum p (c U^V) = (sum p c) U^V
    exactly; §5.3: one softmax over content + RoPE scores with scale
    1/sqrt(d_c' + d_R).  Absorbed oracle (+ library matmuls for q~ and z U^V)
    must equal the explicit per-head expansion to 1e-12."""
    rng = np.random.default_rng(13)
    B, H, d_c, d_h, d_v, T = 2, 3, 16, 8, 6, 75
    latent, q_c, q_r, U_K, U_V = _mla_problem(rng, B, H, d_c, d_r, d_h, d_v, T)
    cache, table = _paged_latent(latent, perm_seed=2)
    lens = np.array([75, 13])
    scale = 1.0 / math.sqrt(d_h + d_r)
    o_explicit = orc.mla_explicit(q_c, q_r, cache, lens, table, U_K, U_V,
                                  scale)
    q_tilde = orc.mla_absorb_q(q_c, U_K)              # q^C (U^K_h)^T
    z = orc.decode_mla(q_tilde, q_r, cache, lens, table, scale)
    o_absorbed = orc.mla_project_out(z, U_V)          # z U^V_h
    np.testing.assert_allclose(o_absorbed, o_explicit, rtol=0, atol=1e-12)


def test_mla_rope_branch_changes_scores():
    """The decoupled RoPE branch contributes to the scores only (HEADS §5.3):
    zeroing k^R changes the result, zeroing the rope columns of the output
    is impossible since z is d_c wide."""
    rng = np.random.default_rng(14)
    B, H, d_c, d_r, T = 1, 2, 8, 4, 40
    latent = rng.standard_normal((B, T, d_c + d_r))
    cache, table = _paged_latent(latent)
    q_l = rng.standard_normal((B, H, d_c))
    q_r = rng.standard_normal((B, H, d_r)) * 3
    z = orc.decode_mla(q_l, q_r, cache, np.array([T]), table, 0.3)
    assert z.shape == (B, H, d_c)
    cache0 = cache.copy()
    cache0[..., d_c:] = 0
    z0 = orc.decode_mla(q_l, q_r, cache0, np.array([T]), table, 0.3)
    assert np.abs(z - z0).max() > 1e-3


def test_mla_matches_dense_library_softmax():
    rng = np.random.default_rng(15)
    B, H, d_c, d_r, T = 2, 4, 32, 8, 130
    latent = rng.standard_normal((B, T, d_c + d_r))
    cache, table = _paged_latent(latent, perm_seed=9)
    q_l = rng.standard_normal((B, H, d_c))
    q_r = rng.standard_normal((B, H, d_r))
    lens = np.array([130, 64])
    z = orc.decode_mla(q_l, q_r, cache, lens, table, 0.1)
    for b in range(B):
        n = lens[b]
        C, KR = latent[b, :n, :d_c], latent[b, :n, d_c:]
        for h in range(H):
            p = scipy.special.softmax(0.1 * (C @ q_l[b, h] + KR @ q_r[b, h]))
            np.testing.assert_allclose(z[b, h], p @ C, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------- bytes model
def test_cache_bytes_closed_form_matches_page_table():
    g = _golden("cache_bytes.json")
    MiB, GiB, KiB = 2.0 ** 20, 2.0 ** 30, 2.0 ** 10
    for row in g["kv_per_layer_MiB"]:
        got = orc.bytes_kv(row["B"], row["T"], row["H_kv"], row["d"], row["s"])
        assert got == row["MiB"] * MiB
    r = g["kv_32_layers_GiB"]
    assert orc.bytes_kv(r["B"], r["T"], r["H_kv"], r["d"], r["s"]) * \
        r["layers"] == r["GiB"] * GiB
    m = g["mla"]
    lat = orc.bytes_mla(m["B"], m["T"], m["r"], m["d_R"], m["s"])
    assert lat / (m["B"] * m["T"] * m["s"]) == m["latent_elems_per_token"]
    expanded = m["H"] * (m["d_c_head"] + m["d_R"] + m["d_v"])
    assert expanded == m["expanded_elems_per_token"]
    assert round(expanded / m["latent_elems_per_token"], 1) == m["ratio_approx"]
    assert round(lat / MiB) == m["latent_MiB_approx"]
    assert round(m["B"] * m["T"] * expanded * m["s"] / GiB, 1) == \
        m["expanded_GiB_approx"]
    for row in g["per_token_per_layer_KiB"]:
        assert orc.bytes_kv(1, 1, row["H_kv"], row["d"], row["s"]) == \
            row["KiB"] * KiB


def test_workload_block_tables_are_permutations():
    """The seeded generator's tables index every owned block exactly once."""
    g = torch.Generator().manual_seed(0)
    lens = [1, 64, 65, 1000]
    table, nblk = make_block_table(lens, g)
    ids = table[table >= 0].tolist()
    assert sorted(ids) == list(range(nblk))
    assert [(table[b] >= 0).sum().item() for b in range(4)] == [1, 1, 2, 16]


# ------------------------------------------- global (sink) tokens, ring table
def _contiguous_case(rng, H_q, H_kv, d, T):
    """One sequence with an identity block table: the cache holds keys
    0..T-1 in order, so rows can also be selected directly."""
    nb = (T + 63) // 64
    q = rng.standard_normal((1, H_q, d))
    k = rng.standard_normal((nb, H_kv, 64, d))
    v = rng.standard_normal((nb, H_kv, 64, d))
    table = np.arange(nb, dtype=np.int32)[None, :]
    return q, k, v, table


def test_vis_without_sink_or_ring_is_decode_gqa():
    """Sink 0 and no ring: the same keys in the same order as the plain
    decode, so the results are bit-identical (with and without a window)."""
    rng = np.random.default_rng(31)
    q, k, v, table = _contiguous_case(rng, 4, 2, 16, 300)
    for w in (0, 1, 70, 299, 5000):
        a = orc.decode_gqa(q, k, v, np.array([300], dtype=np.int32), table, 0.2, window=w)
        b = orc.decode_gqa_vis(q, k, v, np.array([300], dtype=np.int32), table, 0.2, window=w, sink=0, ring=0)
        assert np.array_equal(a, b), w


def test_vis_window_plus_sink_selects_those_keys():
    """Window w=5 and sink g=3 at T=20: exactly keys {0,1,2} and {15..19}
    carry weight (attention-head §3, window plus global tokens), and the
    output is the softmax over just those rows, computed directly."""
    rng = np.random.default_rng(32)
    q, k, v, table = _contiguous_case(rng, 2, 1, 8, 20)
    out, p = orc.decode_gqa_vis(q, k, v, np.array([20], dtype=np.int32), table, 0.7, window=5, sink=3,
                                return_probs=True)
    for h in range(2):
        assert set(np.nonzero(p[0, h])[0].tolist()) == {0, 1, 2, 15, 16, 17, 18, 19}
        assert abs(p[0, h].sum() - 1.0) < 1e-12
    rows = [0, 1, 2, 15, 16, 17, 18, 19]
    K = k[0, 0, rows]
    V = v[0, 0, rows]
    for h in range(2):
        s = 0.7 * K @ q[0, h]
        e = np.exp(s - s.max())
        np.testing.assert_allclose(out[0, h], (e / e.sum()) @ V, rtol=0, atol=1e-12)


def test_vis_sink_covering_all_keys_is_full_attention():
    rng = np.random.default_rng(33)
    q, k, v, table = _contiguous_case(rng, 4, 4, 8, 150)
    full = orc.decode_gqa(q, k, v, np.array([150], dtype=np.int32), table, 0.3, window=0)
    got = orc.decode_gqa_vis(q, k, v, np.array([150], dtype=np.int32), table, 0.3, window=10, sink=150)
    np.testing.assert_allclose(got, full, rtol=0, atol=1e-12)


def test_vis_ring_table_reads_the_same_rows():
    """A ring table whose slots hold the blocks the window (and the sink)
    reach gives exactly the result of the full, identity-table cache: the
    ring only changes where the rows live.  Sink 10 keeps slot 0; the window
    blocks 9 and 10 of T=700, w=100 live in slots 1 + i % 3."""
    rng = np.random.default_rng(34)
    T, w, g, R = 700, 100, 10, 3
    q, k, v, table = _contiguous_case(rng, 4, 2, 16, T)
    ref = orc.decode_gqa_vis(q, k, v, np.array([T], dtype=np.int32), table, 0.25, window=w, sink=g)
    A = 1
    slots = A + R
    kr = rng.standard_normal((slots + 2, 2, 64, 16))     # unused blocks hold noise
    vr = rng.standard_normal((slots + 2, 2, 64, 16))
    ring_table = np.array([[5, 2, 0, 4]], dtype=np.int32)  # slot -> physical block
    for logical in [0, 9, 10]:
        slot = logical if logical < A else A + logical % R
        kr[ring_table[0, slot]] = k[logical]
        vr[ring_table[0, slot]] = v[logical]
    got = orc.decode_gqa_vis(q, kr, vr, np.array([T], dtype=np.int32), ring_table, 0.25, window=w, sink=g, ring=R)
    assert np.array_equal(got, ref)


def _visible_keys(p):
    return [set(np.nonzero(p[b, h])[0].tolist()) for b in range(p.shape[0])
            for h in range(p.shape[1])]


def test_vis_global_set_matches_page_figure():
    """The attention-head §3 figure (right panel): w=3, G={0,5}.  The decode
    query of a sequence with T keys is row T-1: row 8 sees {0,5,6,7,8}, the
    global row 5 sees all of 0..5 (fixture tests/golden/global_tokens.json)."""
    fx = json.load(open(os.path.join(GOLDEN, "global_tokens.json")))
    rng = np.random.default_rng(35)
    for case in fx["cases"]:
        T = case["T"]
        q, k, v, table = _contiguous_case(rng, 2, 1, 8, T)
        gp = np.array([fx["global"]], dtype=np.int32)
        _, p = orc.decode_gqa_vis(q, k, v, np.array([T], dtype=np.int32), table, 0.5,
                                  window=fx["window"], global_pos=gp, return_probs=True)
        assert all(ks == set(case["visible"]) for ks in _visible_keys(p)), T


def test_vis_global_set_brute_force_membership():
    """Every (T, G) over small cases: exactly the keys the definition lists
    carry weight -- window, global keys, and everything for a global query;
    a -1 pad or an entry that does not ascend ends the row."""
    rng = np.random.default_rng(36)
    for T in range(1, 20):
        for row in ([0, 5], [3], [T - 1], [2, 9, 11, -1, -1], [4, 7, 6, 12], [-1, 3]):
            w = 3
            q, k, v, table = _contiguous_case(rng, 1, 1, 4, T)
            gp = np.array([row], dtype=np.int32)
            _, p = orc.decode_gqa_vis(q, k, v, np.array([T], dtype=np.int32), table, 0.5,
                                      window=w, global_pos=gp, return_probs=True)
            G, prev = set(), -1
            for x in row:
                if x <= prev:
                    break
                G.add(x)
                prev = x
            if (T - 1) in G:
                want = set(range(T))
            else:
                want = {j for j in range(T) if j >= T - w or j in G}
            assert _visible_keys(p)[0] == want, (T, row)


def test_vis_global_prefix_equals_sink_tokens():
    """G = {0..g-1} is the sink prefix: same keys, same order, bit-identical
    (attention-head §3, window plus global tokens)."""
    rng = np.random.default_rng(37)
    q, k, v, table = _contiguous_case(rng, 4, 2, 16, 500)
    lens = np.array([500], dtype=np.int32)
    for g in (1, 7, 64, 70):
        a = orc.decode_gqa_vis(q, k, v, lens, table, 0.2, window=100, sink=g)
        gp = np.arange(g, dtype=np.int32)[None, :]
        b = orc.decode_gqa_vis(q, k, v, lens, table, 0.2, window=100, global_pos=gp)
        assert np.array_equal(a, b), g


@pytest.mark.parametrize("T,w,g,R", [(700, 100, 10, 3), (65, 64, 0, 2), (1000, 200, 70, 5),
                                     (129, 1, 0, 1), (5000, 640, 64, 11), (300, 63, 130, 2)])
def test_vis_ring_table_any_geometry_reads_the_same_rows(T, w, g, R):
    """For any ring large enough for the window (R * 64 >= w + 63), a table
    row of A sink slots + R ring slots holding the sink blocks and the blocks
    the window reaches gives the full table's result bit for bit; every other
    block of the ring-side pool holds noise that must never be read."""
    if R * 64 < w + 63:
        pytest.skip("ring smaller than the window")
    rng = np.random.default_rng(T + w + g + R)
    q, k, v, table = _contiguous_case(rng, 2, 1, 8, T)
    lens = np.array([T], dtype=np.int32)
    ref = orc.decode_gqa_vis(q, k, v, lens, table, 0.3, window=w, sink=g)
    A = (g + 63) // 64
    nb = (T + 63) // 64
    lo_blk = max(0, T - w) // 64
    slots = A + R
    perm = rng.permutation(slots + 3).astype(np.int32)
    ring_table = perm[:slots][None, :]
    kr = rng.standard_normal((slots + 3, 1, 64, 8))
    vr = rng.standard_normal((slots + 3, 1, 64, 8))
    needed = set(range(min(A, nb))) | set(range(lo_blk, nb))
    for logical in needed:
        slot = logical if logical < A else A + logical % R
        kr[ring_table[0, slot]] = k[logical]
        vr[ring_table[0, slot]] = v[logical]
    got = orc.decode_gqa_vis(q, kr, vr, lens, ring_table, 0.3, window=w, sink=g, ring=R)
    assert np.array_equal(got, ref)


def _global_ring_table(rng, k, v, T, w, R, gp_row, spare=3):
    """Table row of n_g global slots + R ring slots for one sequence whose
    full-table cache is (k, v): global slot k names the block of position
    gp_row[k] (positions sharing a block share its physical block), ring
    slot n_g + i % R names logical block i for the blocks the window
    reaches.  Every physical block nothing names holds noise."""
    n_g = len(gp_row)
    nb = (T + 63) // 64
    w0 = max(0, T - w) // 64
    gblocks = sorted({p // 64 for p in gp_row if p >= 0})
    n_phys = len(gblocks) + R + spare
    perm = rng.permutation(n_phys).astype(np.int32)
    table = np.full((1, n_g + R), -1, dtype=np.int32)
    kr = rng.standard_normal((n_phys,) + k.shape[1:])
    vr = rng.standard_normal((n_phys,) + v.shape[1:])
    phys_of = {}
    for j, blk in enumerate(gblocks):
        phys_of[blk] = perm[j]
        kr[perm[j]] = k[blk]
        vr[perm[j]] = v[blk]
    for kk, pos in enumerate(gp_row):
        if pos >= 0:
            table[0, kk] = phys_of[pos // 64]
    for i in range(w0, nb):
        ph = perm[len(gblocks) + i % R]
        table[0, n_g + i % R] = ph
        kr[ph] = k[i]
        vr[ph] = v[i]
    return kr, vr, table


@pytest.mark.parametrize("T,w,R,gp", [
    (9, 3, 2, [0, 5]),                      # the §3 figure's G = {0, 5}, w = 3
    (700, 100, 3, [0, 5, 130, 131, 640]),   # two positions share a block; one in the window
    (1000, 200, 5, [63, 64, 799, 801]),     # 799 straddles the window's first block
    (5000, 640, 11, [1, 2, 3, 4000, 4500, -1, -1]),
    (129, 1, 1, [0, 127]),
    (300, 63, 2, [10, 250, 298]),
])
def test_vis_global_set_ring_reads_the_same_rows(T, w, R, gp):
    """A window layer that keeps the positions of an explicit global set G
    (attention-head article, §3): a table row of n_g global slots + a ring
    holding the window's blocks gives the full table's result bit for bit,
    wherever G's positions lie (before the window, in its first block, in
    it), and no other physical block is read."""
    if R * 64 < w + 63:
        pytest.skip("ring smaller than the window")
    gp_row = list(gp)
    if (T - 1) in gp_row and T > w:
        pytest.skip("a global query needs the whole history")
    rng = np.random.default_rng(T + 7 * w + R)
    q, k, v, table = _contiguous_case(rng, 2, 1, 8, T)
    lens = np.array([T], dtype=np.int32)
    gpos = np.array([gp_row], dtype=np.int32)
    ref = orc.decode_gqa_vis(q, k, v, lens, table, 0.3, window=w, global_pos=gpos)
    kr, vr, ring_table = _global_ring_table(rng, k, v, T, w, R, gp_row)
    got = orc.decode_gqa_vis(q, kr, vr, lens, ring_table, 0.3, window=w, ring=R,
                             global_pos=gpos)
    assert np.array_equal(got, ref)


def test_vis_global_set_ring_noise_changes_result_when_a_global_block_is_lost():
    """Negative control of the ring pin: if a global slot names a noise block
    instead of its position's block, the result changes -- the ring layout
    really reads the global slots."""
    T, w, R, gp_row = 700, 100, 3, [0, 5, 130]
    rng = np.random.default_rng(3)
    q, k, v, table = _contiguous_case(rng, 2, 1, 8, T)
    lens = np.array([T], dtype=np.int32)
    gpos = np.array([gp_row], dtype=np.int32)
    ref = orc.decode_gqa_vis(q, k, v, lens, table, 0.3, window=w, global_pos=gpos)
    kr, vr, ring_table = _global_ring_table(rng, k, v, T, w, R, gp_row, spare=3)
    ring_table[0, 2] = kr.shape[0] - 1          # block of position 130 -> a noise block
    got = orc.decode_gqa_vis(q, kr, vr, lens, ring_table, 0.3, window=w, ring=R,
                             global_pos=gpos)
    assert not np.allclose(got, ref)


def test_vis_global_query_with_ring_is_refused():
    """A global query sees the whole history (§3), which a ring no longer
    holds once T > window: the oracle refuses it; with T <= window the
    window covers everything and the call is served."""
    rng = np.random.default_rng(5)
    q, k, v, table = _contiguous_case(rng, 2, 1, 8, 200)
    gpos = np.array([[3, 199]], dtype=np.int32)          # T - 1 = 199 is global
    with pytest.raises(RuntimeError):
        orc.decode_gqa_vis(q, k, v, np.array([200], dtype=np.int32), table, 0.3, window=100,
                           ring=4, global_pos=gpos)
    kr, vr, ring_table = _global_ring_table(rng, k, v, 200, 300, 6, [3, 199])
    ok = orc.decode_gqa_vis(q, kr, vr, np.array([200], dtype=np.int32), ring_table, 0.3,
                            window=300, ring=6, global_pos=gpos)
    full = orc.decode_gqa(q, k, v, np.array([200], dtype=np.int32), table, 0.3, window=0)
    assert np.array_equal(ok, full)


# ------------------------------------------------------- fp8 (E4M3) KV cache
def test_e4m3_values_match_the_format():
    """Closed forms of the OCP FP8 E4M3 format: bias 7, 3 mantissa bits,
    subnormals m/8 * 2^-6, largest finite 448, S.1111.111 NaN."""
    t = orc.e4m3_table()
    assert t[0x00] == 0.0 and t[0x38] == 1.0 and t[0xB8] == -1.0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x08] == 2.0 ** -6 and t[0x01] == 2.0 ** -9 and t[0x07] == 7 * 2.0 ** -9
    assert t[0x40] == 2.0 and t[0x3F] == 1.875
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.sum(np.isnan(t)) == 2


def test_e4m3_encode_round_trip_ties_and_saturation():
    t = orc.e4m3_table()
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert orc.e4m3_encode(t[c]) == c, hex(c)
    assert orc.e4m3_encode(1.0625) == 0x38      # tie 1.0 / 1.125 -> even mantissa
    assert orc.e4m3_encode(1.1875) == 0x3A      # tie 1.125 / 1.25 -> 1.25
    assert orc.e4m3_encode(1.9375) == 0x40      # tie across the binade -> 2.0
    assert orc.e4m3_encode(1000.0) == 0x7E and orc.e4m3_encode(-1000.0) == 0xFE
    assert orc.e4m3_encode(460.0) == 0x7E       # past 448 saturates


def test_quantize_rows_error_bound():
    """Each row's largest element maps to 448 (within rounding) and every
    element is reproduced to e4m3's half-ulp: relative 2^-4 for normals,
    absolute 2^-10 * scale below the normal range."""
    rng = np.random.default_rng(40)
    x = (rng.standard_normal((50, 128)) * rng.uniform(0.01, 30, (50, 1))).astype(np.float32)
    x[7] = 0.0                                        # a zero row
    codes, scales = orc.quantize_rows_e4m3(x)
    assert scales[7] == 0.0 and not codes[7].any()
    deq = orc.dequantize_e4m3(codes, scales)
    amax = np.abs(x).max(axis=1)
    for r in range(50):
        if amax[r] == 0:
            continue
        assert abs(np.abs(deq[r]).max() - amax[r]) <= 1e-6 * amax[r]
        err = np.abs(deq[r] - x[r])
        bound = np.maximum(np.abs(x[r]) * 2.0 ** -4, scales[r] * 2.0 ** -10) * (1 + 1e-6)
        assert np.all(err <= bound), r
