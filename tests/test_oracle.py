"""Pins for the CPU oracle: values the pages print, closed forms, invariants the
pages fix and brute force on tiny inputs.  Each pin is chosen so that a
plausible slip in the oracle (a transposed operand, a wrong group index, a
missing max-subtraction, a dropped mask, appending after attending) fails at
least one of them.  CPU only."""
import math

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import dot_product_attention, oracle_decode, oracle_decode_step, oracle_kv_append
from grouped_query_attention_mqa_b200.workloads import WORKLOADS, kv_cache_bytes


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _two_key_problem(g_read):
    k1, k2 = g_read["k1"], g_read["k2"]
    q1, q2 = g_read["q1"], g_read["q2"]
    v1, v2 = g_read["v1"], g_read["v2"]
    q = np.array([[q1, q2]], dtype=np.float64)                # [b=1, h=2, d=2]
    K = np.array([[[k1], [k2]]], dtype=np.float64)            # [1, m=2, g=1, 2]
    V = np.array([[[v1], [v2]]], dtype=np.float64)
    return q, K, V


# ------------------------------------------------------------ printed examples

def test_worked_example_two_keys_scale_one(golden):
    """Study notes §4: two heads over one shared K pick opposite positions; the
    exact weights are sigmoid(3) and 1 - sigmoid(3)."""
    g = golden("worked_example_two_keys.txt")
    q, K, V = _two_key_problem(g)
    o, lse, w = oracle_decode(q, K, V, [2], g=1, scale=1.0, return_weights=True)
    np.testing.assert_allclose(w[0][0], g["scale_1.head1"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(w[0][1], g["scale_1.head2"], rtol=0, atol=1e-15)
    # V is the identity, so each output row is the weight row
    np.testing.assert_allclose(o[0], w[0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], g["scale_1.lse"] * 2, rtol=0, atol=1e-14)
    assert w[0][0][0] > 0.5 and w[0][1][1] > 0.5


def test_worked_example_two_keys_scaled(golden):
    g = golden("worked_example_two_keys.txt")
    q, K, V = _two_key_problem(g)
    o, _, w = oracle_decode(q, K, V, [2], g=1, scale=1 / math.sqrt(2.0), return_weights=True)
    np.testing.assert_allclose(w[0][0], g["scale_rsqrt2.head1"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(w[0][1], g["scale_rsqrt2.head2"], rtol=0, atol=1e-15)


def test_worked_example_brute_force(golden):
    """The per-query DotProductAttention of the review's §2.1 on the same example."""
    g = golden("worked_example_two_keys.txt")
    K = np.array([g["k1"], g["k2"]])
    V = np.array([g["v1"], g["v2"]])
    y, w = dot_product_attention(g["q1"], K, V, scale=1.0)
    np.testing.assert_allclose(w, g["scale_1.head1"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(y, g["scale_1.head1"], rtol=0, atol=1e-15)
    y, w = dot_product_attention(g["q2"], K, V, scale=1.0)
    np.testing.assert_allclose(w, g["scale_1.head2"], rtol=0, atol=1e-15)


def test_shape_example(golden):
    """Study notes §2: L_q=4, L_k=6, d_h=128 give scores [4,6] and output [4,128]
    (four query heads of one sequence reading one shared K/V)."""
    s = golden("shape_example.txt")
    Lq, Lk, dh = int(s["L_q"][0]), int(s["L_k"][0]), int(s["d_h"][0])
    rng = np.random.default_rng(0)
    o, lse, w = oracle_decode(_rand(rng, 1, Lq, dh), _rand(rng, 1, Lk, 1, dh), _rand(rng, 1, Lk, 1, dh),
                              [Lk], g=1, scale=1 / math.sqrt(dh), return_weights=True)
    assert list(w[0].shape) == [int(x) for x in s["scores_shape"]]
    assert list(o[0].shape) == [int(x) for x in s["output_shape"]]


# ------------------------------------------------------------ brute force

@pytest.mark.parametrize("h,g", [(4, 1), (4, 2), (4, 4), (6, 3)])
def test_oracle_matches_per_head_brute_force(h, g):
    """Every (sequence, head) of the batched oracle equals DotProductAttention
    (Python loops) over that head's K/V group j(i) = i // (h/g)."""
    rng = np.random.default_rng(h * 10 + g)
    b, m_max, dk, dv = 3, 7, 5, 3
    lens = [1, 4, 7]
    q = _rand(rng, b, h, dk)
    K = _rand(rng, b, m_max, g, dk)
    V = _rand(rng, b, m_max, g, dv)
    scale = 0.7
    o, lse = oracle_decode(q, K, V, lens, g=g, scale=scale)
    for bi in range(b):
        L = lens[bi]
        for i in range(h):
            j = i // (h // g)
            y, w = dot_product_attention(q[bi, i], K[bi, :L, j], V[bi, :L, j], scale=scale)
            np.testing.assert_allclose(o[bi, i], y, rtol=0, atol=1e-13)
            logits = [scale * float(np.dot(q[bi, i], K[bi, t, j])) for t in range(L)]
            top = max(logits)
            ref_lse = top + math.log(math.fsum(math.exp(x - top) for x in logits))
            assert abs(lse[bi, i] - ref_lse) < 1e-12


# ------------------------------------------------------------ invariants

def test_mqa_equals_mha_with_replicated_kv():
    """Multi-Query Attention page, "从 MHA 到 MQA": every Q_i attends to the one
    shared K/V, so MQA is MHA whose h K/V heads are h copies of the shared one."""
    rng = np.random.default_rng(1)
    b, h, m, d = 2, 8, 9, 6
    q = _rand(rng, b, h, d)
    K = _rand(rng, b, m, 1, d)
    V = _rand(rng, b, m, 1, d)
    lens = [5, 9]
    o1, l1 = oracle_decode(q, K, V, lens, g=1, scale=0.3)
    oh, lh = oracle_decode(q, np.repeat(K, h, axis=2), np.repeat(V, h, axis=2), lens, g=h, scale=0.3)
    np.testing.assert_allclose(o1, oh, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l1, lh, rtol=0, atol=1e-14)


def test_gqa_is_mqa_per_group():
    """GQA blog, "第三站: GQA": H query heads in G groups, each group sharing one
    K/V head.  Group j's heads equal an MQA call over that group's K/V alone;
    this fixes contiguous grouping (head i -> group i // (h/g))."""
    rng = np.random.default_rng(2)
    b, h, g, m, d = 2, 8, 4, 6, 5
    q = _rand(rng, b, h, d)
    K = _rand(rng, b, m, g, d)
    V = _rand(rng, b, m, g, d)
    lens = [6, 3]
    o, lse = oracle_decode(q, K, V, lens, g=g, scale=0.5)
    hq = h // g
    for j in range(g):
        oj, lj = oracle_decode(q[:, j * hq:(j + 1) * hq], K[:, :, j:j + 1], V[:, :, j:j + 1], lens, g=1, scale=0.5)
        np.testing.assert_allclose(o[:, j * hq:(j + 1) * hq], oj, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[:, j * hq:(j + 1) * hq], lj, rtol=0, atol=1e-14)


def test_gqa_h_is_mha_and_gqa_1_is_mqa():
    """GQA-H (one head per group) equals the per-head incremental MHA of the
    review's §2.4 (K/V [b,h,m,k]); GQA-1 equals the single shared head."""
    rng = np.random.default_rng(3)
    b, h, m, d = 2, 4, 5, 3
    q = _rand(rng, b, h, d)
    K_mha = _rand(rng, b, h, m, d)          # the review's prev_K layout [b, h, m, k]
    V_mha = _rand(rng, b, h, m, d)
    o, _ = oracle_decode(q, K_mha.transpose(0, 2, 1, 3), V_mha.transpose(0, 2, 1, 3), [m, m], g=h, scale=1.0)
    for bi in range(b):
        for i in range(h):
            y, _ = dot_product_attention(q[bi, i], K_mha[bi, i], V_mha[bi, i])
            np.testing.assert_allclose(o[bi, i], y, rtol=0, atol=1e-13)
    K1 = K_mha[:, :1].transpose(0, 2, 1, 3)
    V1 = V_mha[:, :1].transpose(0, 2, 1, 3)
    o1, _ = oracle_decode(q, K1, V1, [m, m], g=1, scale=1.0)
    for bi in range(b):
        for i in range(h):
            y, _ = dot_product_attention(q[bi, i], K_mha[bi, 0], V_mha[bi, 0])
            np.testing.assert_allclose(o1[bi, i], y, rtol=0, atol=1e-13)


@settings(max_examples=25, deadline=None)
@given(hq=st.sampled_from([1, 2, 4]), g=st.sampled_from([1, 2, 3]), L=st.integers(1, 12), seed=st.integers(0, 10**6))
def test_weights_sum_to_one_and_match_lse(hq, g, L, seed):
    """Softmax weights over the valid rows sum to one, and w_t = exp(s_t - lse)."""
    rng = np.random.default_rng(seed)
    h, d = hq * g, 4
    q = _rand(rng, 1, h, d)
    K = _rand(rng, 1, 12, g, d)
    V = _rand(rng, 1, 12, g, d)
    _, lse, w = oracle_decode(q, K, V, [L], g=g, scale=1.3, return_weights=True)
    np.testing.assert_allclose(w[0].sum(axis=1), 1.0, rtol=0, atol=1e-13)
    for i in range(h):
        s = 1.3 * (K[0, :L, i // hq] @ q[0, i])
        np.testing.assert_allclose(np.exp(s - lse[0, i]), w[0][i], rtol=1e-12, atol=1e-15)


@settings(max_examples=25, deadline=None)
@given(hq=st.sampled_from([1, 3]), g=st.sampled_from([1, 2]), dk=st.sampled_from([2, 5]),
       dv=st.sampled_from([1, 3, 6]), L=st.integers(1, 10), seed=st.integers(0, 10**6))
def test_output_is_a_convex_combination_of_the_valid_v_rows(hq, g, dk, dv, L, seed):
    """Each output is a weighted mean of its group's valid V rows, so every
    column lies between that column's minimum and maximum over those rows,
    whatever d_k and d_v are; rows past the length hold values far outside the
    range and must not pull the output out of it."""
    rng = np.random.default_rng(seed)
    h, m = hq * g, 12
    q = _rand(rng, 2, h, dk) * 3.0
    K = _rand(rng, 2, m, g, dk)
    V = _rand(rng, 2, m, g, dv)
    V[:, L:] = 1e6
    o, _ = oracle_decode(q, K, V, [L, L], g=g, scale=0.9)
    assert o.shape == (2, h, dv)
    for bi in range(2):
        for i in range(h):
            rows = V[bi, :L, i // hq]
            assert np.all(o[bi, i] >= rows.min(axis=0) - 1e-12)
            assert np.all(o[bi, i] <= rows.max(axis=0) + 1e-12)


def test_length_one_cache_returns_v():
    """A softmax over one row is 1, so each head's output is that row of V."""
    rng = np.random.default_rng(4)
    b, h, g, m, d = 3, 6, 2, 4, 5
    q = _rand(rng, b, h, d)
    K = _rand(rng, b, m, g, d)
    V = _rand(rng, b, m, g, d)
    o, _ = oracle_decode(q, K, V, [1, 1, 1], g=g, scale=1.0)
    for bi in range(b):
        for i in range(h):
            np.testing.assert_allclose(o[bi, i], V[bi, 0, i // 3], rtol=0, atol=1e-15)


def test_identical_keys_return_mean_of_v():
    """Equal keys give equal logits, hence uniform weights: o = mean of the valid
    V rows and lse = s + log(L)."""
    rng = np.random.default_rng(5)
    b, h, m, d, L = 1, 4, 10, 6, 7
    q = _rand(rng, b, h, d)
    row = _rand(rng, d)
    K = np.broadcast_to(row, (b, m, 1, d)).copy()
    V = _rand(rng, b, m, 1, d)
    o, lse = oracle_decode(q, K, V, [L], g=1, scale=0.9)
    for i in range(h):
        np.testing.assert_allclose(o[0, i], V[0, :L, 0].mean(axis=0), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[0, i], 0.9 * float(q[0, i] @ row) + math.log(L), rtol=0, atol=1e-13)


def test_masked_rows_are_never_read():
    """Rows at t >= lens[b] hold NaN; the result is finite and equals the same
    call on a cache cut to the valid rows."""
    rng = np.random.default_rng(6)
    b, h, g, m, d = 2, 4, 2, 8, 3
    q = _rand(rng, b, h, d)
    K = _rand(rng, b, m, g, d)
    V = _rand(rng, b, m, g, d)
    lens = [3, 8]
    Kn, Vn = K.copy(), V.copy()
    Kn[0, 3:] = np.nan
    Vn[0, 3:] = np.nan
    o, _ = oracle_decode(q, Kn, Vn, lens, g=g, scale=1.0)
    assert np.isfinite(o).all()
    o0, _ = oracle_decode(q[:1], K[:1, :3], V[:1, :3], [3], g=g, scale=1.0)
    np.testing.assert_allclose(o[0], o0[0], rtol=0, atol=1e-15)


def test_large_logits_are_stable_and_pick_the_argmax():
    """With logits ~1e4 apart the softmax is one-hot: o is the V row of the
    largest logit (an implementation without max-subtraction overflows)."""
    rng = np.random.default_rng(7)
    m, d = 6, 4
    K = _rand(rng, 1, m, 1, d)
    V = _rand(rng, 1, m, 1, d)
    q = K[:, 4, 0][:, None, :] * 1e4                     # head 0 aligns with row 4
    o, lse = oracle_decode(q, K, V, [m], g=1, scale=1.0)
    s = (K[0, :, 0] @ q[0, 0])
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    np.testing.assert_allclose(o[0, 0], V[0, int(np.argmax(s)), 0], rtol=0, atol=1e-12)


def test_scale_folds_into_q():
    """scale multiplies q·k, so scaling q by c with scale 1 equals scale c."""
    rng = np.random.default_rng(8)
    q = _rand(rng, 2, 4, 8)
    K = _rand(rng, 2, 9, 2, 8)
    V = _rand(rng, 2, 9, 2, 8)
    a, la = oracle_decode(q * 0.25, K, V, [9, 4], g=2, scale=1.0)
    c, lc = oracle_decode(q, K, V, [9, 4], g=2, scale=0.25)
    np.testing.assert_allclose(a, c, rtol=0, atol=1e-14)
    np.testing.assert_allclose(la, lc, rtol=0, atol=1e-14)


def test_row_permutation_and_v_linearity():
    """Permuting the valid rows of K and V together leaves o unchanged (the
    weighted sum does not depend on row order), and o is linear in V (the
    weights do not depend on V)."""
    rng = np.random.default_rng(9)
    b, h, m, d = 1, 4, 7, 5
    q = _rand(rng, b, h, d)
    K = _rand(rng, b, m, 1, d)
    V1 = _rand(rng, b, m, 1, d)
    V2 = _rand(rng, b, m, 1, d)
    perm = rng.permutation(m)
    o, _ = oracle_decode(q, K, V1, [m], g=1, scale=0.6)
    op, _ = oracle_decode(q, K[:, perm], V1[:, perm], [m], g=1, scale=0.6)
    np.testing.assert_allclose(o, op, rtol=0, atol=1e-14)
    os_, _ = oracle_decode(q, K, V1 + V2, [m], g=1, scale=0.6)
    o2, _ = oracle_decode(q, K, V2, [m], g=1, scale=0.6)
    np.testing.assert_allclose(os_, o + o2, rtol=0, atol=1e-13)


def test_zero_length_gives_zero_row():
    rng = np.random.default_rng(10)
    o, lse = oracle_decode(_rand(rng, 2, 2, 3), _rand(rng, 2, 4, 1, 3), _rand(rng, 2, 4, 1, 3), [0, 2], g=1, scale=1.0)
    assert (o[0] == 0).all() and np.isneginf(lse[0]).all()
    assert np.isfinite(o[1]).all()


# ------------------------------------------------------------ append

def test_append_is_the_concat_of_the_review():
    """The review's §3 step builds new_K = concat(prev_K, k_new): after writing
    at row L the first L+1 rows are that concatenation, bit for bit, and no
    other element changes."""
    rng = np.random.default_rng(11)
    b, m, g, d = 3, 6, 2, 4
    Kc = rng.integers(0, 2**16, size=(b, m, g, d), dtype=np.uint16)
    Vc = rng.integers(0, 2**16, size=(b, m, g, d), dtype=np.uint16)
    kn = rng.integers(0, 2**16, size=(b, g, d), dtype=np.uint16)
    vn = rng.integers(0, 2**16, size=(b, g, d), dtype=np.uint16)
    pos = np.array([0, 3, 5])
    Kc0, Vc0 = Kc.copy(), Vc.copy()
    K2, V2 = oracle_kv_append(Kc, Vc, kn, vn, pos)
    for bi in range(b):
        L = pos[bi]
        cat_k = np.concatenate([Kc[bi, :L], kn[bi][None]], axis=0)
        cat_v = np.concatenate([Vc[bi, :L], vn[bi][None]], axis=0)
        assert np.array_equal(K2[bi, :L + 1], cat_k) and np.array_equal(V2[bi, :L + 1], cat_v)
        assert np.array_equal(K2[bi, L + 1:], Kc[bi, L + 1:]) and np.array_equal(V2[bi, L + 1:], Vc[bi, L + 1:])
    assert np.array_equal(Kc, Kc0) and np.array_equal(Vc, Vc0)   # inputs untouched (copy semantics)


def test_append_out_of_range_row_writes_nothing():
    rng = np.random.default_rng(12)
    Kc = rng.standard_normal((2, 3, 1, 2))
    kn = rng.standard_normal((2, 1, 2))
    K2, V2 = oracle_kv_append(Kc, Kc, kn, kn, [3, -1])
    assert np.array_equal(K2, Kc) and np.array_equal(V2, Kc)


def test_step_appends_before_attending():
    """In the review's §3 the new K/V is concatenated before the logits, so the
    new token attends to itself: a query aligned with a large k_new returns
    v_new (appending after attending would miss it)."""
    rng = np.random.default_rng(13)
    b, h, m, d = 2, 2, 5, 4
    Kc = _rand(rng, b, m, 1, d)
    Vc = _rand(rng, b, m, 1, d)
    kn = _rand(rng, b, 1, d)
    vn = _rand(rng, b, 1, d)
    q = np.repeat(kn, h, axis=1) * 1e3
    o, _, K2, _ = oracle_decode_step(q, Kc, Vc, kn, vn, [2, 4], g=1, scale=1.0)
    for bi in range(b):
        for i in range(h):
            np.testing.assert_allclose(o[bi, i], vn[bi, 0], rtol=0, atol=1e-9)


# ------------------------------------------------------------ cache size

def test_mha_over_mqa_cache_bytes_is_h():
    """Multi-Query Attention page, "为什么能节省 KV Cache": 2·T·n_h·d_h versus
    2·T·d_h, i.e. 1/32 at n_h = 32 — the MHA/MQA workload pair's ratio."""
    mha, mqa = WORKLOADS["mha_b16_m16k"], WORKLOADS["mqa_b16_m16k"]
    a = kv_cache_bytes(mha.b, mha.m_max, mha.g, mha.d_k, mha.d_v, mha.elem_bytes)
    c = kv_cache_bytes(mqa.b, mqa.m_max, mqa.g, mqa.d_k, mqa.d_v, mqa.elem_bytes)
    assert a == 32 * c and a == 4 * 2**30


# ------------------------------------------------------------ local window

def test_window_one_returns_the_newest_row_of_v(golden):
    """Study notes §6.1/§6.4 local attention with a window of one position: the
    softmax has one term, so every head returns V at row L-1 and lse is that
    row's logit.  On the two-key example the window keeps only k2/v2."""
    g = golden("worked_example_two_keys.txt")
    q, K, V = _two_key_problem(g)
    o, lse, w = oracle_decode(q, K, V, [2], g=1, scale=1.0, return_weights=True, window=1)
    np.testing.assert_array_equal(w[0], [[0.0, 1.0], [0.0, 1.0]])
    np.testing.assert_array_equal(o[0], [g["v2"], g["v2"]])
    np.testing.assert_allclose(lse[0], [float(np.dot(g["q1"], g["k2"])), float(np.dot(g["q2"], g["k2"]))],
                               rtol=0, atol=1e-15)


def test_window_covering_the_cache_is_full_attention(golden):
    """A window at least as long as the sequence leaves every row in."""
    g = golden("worked_example_two_keys.txt")
    q, K, V = _two_key_problem(g)
    for window in (2, 3, 100):
        _, _, w = oracle_decode(q, K, V, [2], g=1, scale=1.0, return_weights=True, window=window)
        np.testing.assert_allclose(w[0][0], g["scale_1.head1"], rtol=0, atol=1e-15)
        np.testing.assert_allclose(w[0][1], g["scale_1.head2"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("window", [1, 3, 5, 32])
def test_window_is_brute_force_on_the_newest_rows(window):
    """With window w the result is DotProductAttention over rows L-w .. L-1 only,
    computed by the per-query brute force on that slice; rows before the
    window hold NaN and must not be read."""
    rng = np.random.default_rng(40 + window)
    b, h, g, m, d = 3, 4, 2, 40, 5
    q = _rand(rng, b, h, d)
    K = _rand(rng, b, m, g, d)
    V = _rand(rng, b, m, g, d)
    lens = [40, 7, 2]
    Kn, Vn = K.copy(), V.copy()
    for bi, L in enumerate(lens):
        lo = max(0, L - window)
        Kn[bi, :lo] = np.nan
        Vn[bi, :lo] = np.nan
        Kn[bi, L:] = np.nan
        Vn[bi, L:] = np.nan
    o, lse, w = oracle_decode(q, Kn, Vn, lens, g=g, scale=0.7, return_weights=True, window=window)
    assert np.isfinite(o).all()
    for bi, L in enumerate(lens):
        lo = max(0, L - window)
        assert np.count_nonzero(w[bi]) == h * (L - lo)
        for i in range(h):
            j = i // (h // g)
            y, wi = dot_product_attention(q[bi, i], K[bi, lo:L, j], V[bi, lo:L, j], scale=0.7)
            np.testing.assert_allclose(o[bi, i], y, rtol=0, atol=1e-13)
            np.testing.assert_allclose(w[bi][i, lo:], wi, rtol=0, atol=1e-15)


def test_notes_window_is_current_plus_31_previous():
    """Study notes §6.1: the decoder window is the current position and the 31
    before it, i.e. window=32 attends rows L-32 .. L-1 (exactly 32 of them)."""
    rng = np.random.default_rng(41)
    L = 100
    q = _rand(rng, 1, 2, 4)
    K = _rand(rng, 1, L, 1, 4)
    V = _rand(rng, 1, L, 1, 4)
    _, _, w = oracle_decode(q, K, V, [L], g=1, scale=1.0, return_weights=True, window=32)
    nz = np.nonzero(w[0][0])[0]
    assert nz.min() == L - 32 and nz.max() == L - 1 and len(nz) == 32


def test_step_with_window_attends_the_appended_row():
    """The appended row is the newest one, so it is inside any window: with
    window=1 the step returns the new V row for every head."""
    rng = np.random.default_rng(42)
    b, h, g, m, d = 2, 4, 2, 9, 3
    q = _rand(rng, b, h, d)
    K = _rand(rng, b, m, g, d)
    V = _rand(rng, b, m, g, d)
    kn, vn = _rand(rng, b, g, d), _rand(rng, b, g, d)
    o, _, _, _ = oracle_decode_step(q, K, V, kn, vn, [3, 8], g=g, scale=1.0, window=1)
    for bi in range(b):
        for i in range(h):
            np.testing.assert_array_equal(o[bi, i], vn[bi, i // (h // g)])


# ------------------------------------------------------------ prefill (batched, causal)

from oracle import oracle_prefill   # noqa: E402


def _packed(rng, lens, h, g, d):
    T = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return _rand(rng, T, h, d), _rand(rng, T, g, d), _rand(rng, T, g, d), cu


@pytest.mark.parametrize("h,g", [(4, 1), (4, 2), (4, 4)])
def test_prefill_is_brute_force_over_the_causal_prefix(h, g):
    """Query t of a sequence is DotProductAttention ([velog review] §2.1) over
    keys 0..t of the same sequence: the review's batched form with a causal
    mask."""
    rng = np.random.default_rng(60 + h + g)
    lens = [5, 1, 3]
    q, k, v, cu = _packed(rng, lens, h, g, 3)
    o, _ = oracle_prefill(q, k, v, cu, g=g, scale=0.8)
    for si, n in enumerate(lens):
        a = int(cu[si])
        for t in range(n):
            for i in range(h):
                j = i // (h // g)
                y, _ = dot_product_attention(q[a + t, i], k[a:a + t + 1, j], v[a:a + t + 1, j], scale=0.8)
                np.testing.assert_allclose(o[a + t, i], y, rtol=0, atol=1e-13)


def test_prefill_first_position_returns_its_own_v():
    """The causal mask leaves one key for position 0: o = v[0] exactly."""
    rng = np.random.default_rng(61)
    q, k, v, cu = _packed(rng, [4, 6], 4, 2, 5)
    o, lse = oracle_prefill(q, k, v, cu, g=2, scale=1.3)
    for a in (0, 4):
        for i in range(4):
            np.testing.assert_array_equal(o[a, i], v[a, i // 2])
            np.testing.assert_allclose(lse[a, i], 1.3 * float(q[a, i] @ k[a, i // 2]), rtol=0, atol=1e-13)


def test_prefill_without_mask_sees_the_whole_sequence():
    rng = np.random.default_rng(62)
    lens = [4, 3]
    q, k, v, cu = _packed(rng, lens, 2, 1, 3)
    o, _ = oracle_prefill(q, k, v, cu, g=1, scale=1.0, causal=False)
    for si, n in enumerate(lens):
        a = int(cu[si])
        for t in range(n):
            for i in range(2):
                y, _ = dot_product_attention(q[a + t, i], k[a:a + n, 0], v[a:a + n, 0], scale=1.0)
                np.testing.assert_allclose(o[a + t, i], y, rtol=0, atol=1e-13)


def test_prefill_prefix_is_unchanged_by_later_tokens():
    """Causality: outputs of positions 0..n-1 do not depend on tokens appended
    after them."""
    rng = np.random.default_rng(63)
    q, k, v, cu = _packed(rng, [9], 4, 1, 4)
    o_full, _ = oracle_prefill(q, k, v, cu, g=1, scale=1.0)
    o_cut, _ = oracle_prefill(q[:5], k[:5], v[:5], [0, 5], g=1, scale=1.0)
    np.testing.assert_allclose(o_full[:5], o_cut, rtol=0, atol=1e-15)


def test_prefill_last_position_is_the_decode_step():
    """The last position of a prefill attends to the whole sequence, exactly as
    one decode step over a cache holding that sequence."""
    rng = np.random.default_rng(64)
    lens = [7, 2]
    q, k, v, cu = _packed(rng, lens, 6, 3, 4)
    o, lse = oracle_prefill(q, k, v, cu, g=3, scale=0.5)
    for si, n in enumerate(lens):
        a = int(cu[si])
        od, lsed = oracle_decode(q[a + n - 1][None], k[a:a + n][None], v[a:a + n][None], [n], g=3, scale=0.5)
        np.testing.assert_allclose(o[a + n - 1], od[0], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[a + n - 1], lsed[0], rtol=0, atol=1e-13)


def test_prefill_mqa_equals_mha_with_replicated_kv():
    rng = np.random.default_rng(65)
    q, k, v, cu = _packed(rng, [6, 3], 4, 1, 3)
    o1, _ = oracle_prefill(q, k, v, cu, g=1, scale=1.0)
    o4, _ = oracle_prefill(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), cu, g=4, scale=1.0)
    np.testing.assert_allclose(o1, o4, rtol=0, atol=1e-15)


# ------------------------------------------------------------ beams sharing a prefix

from oracle import oracle_decode_beam   # noqa: E402


def _beam_problem(rng, b, W, h, g, d, mp, ms):
    return (_rand(rng, b, W, h, d), _rand(rng, b, mp, g, d), _rand(rng, b, mp, g, d),
            _rand(rng, b * W, ms, g, d), _rand(rng, b * W, ms, g, d))


def test_beam_is_brute_force_over_prefix_then_suffix():
    """Beam (s, w), head i: DotProductAttention ([velog review] §2.1) over the
    shared prefix rows of sequence s followed by the beam's own suffix rows."""
    rng = np.random.default_rng(70)
    b, W, h, g, d = 2, 3, 4, 2, 3
    q, pk, pv, sk, sv = _beam_problem(rng, b, W, h, g, d, 6, 4)
    lp, ls = [5, 2], [0, 1, 4, 3, 2, 0]
    o, _ = oracle_decode_beam(q, pk, pv, lp, sk, sv, ls, g=g, scale=0.6)
    for si in range(b):
        for w in range(W):
            r = si * W + w
            for i in range(h):
                j = i // (h // g)
                K = np.concatenate([pk[si, :lp[si], j], sk[r, :ls[r], j]])
                V = np.concatenate([pv[si, :lp[si], j], sv[r, :ls[r], j]])
                y, _ = dot_product_attention(q[si, w, i], K, V, scale=0.6)
                np.testing.assert_allclose(o[si, w, i], y, rtol=0, atol=1e-13)


def test_beams_with_the_same_suffix_agree():
    """Beams are independent rows: equal queries and equal suffixes give equal outputs."""
    rng = np.random.default_rng(71)
    q, pk, pv, sk, sv = _beam_problem(rng, 1, 4, 2, 1, 3, 5, 3)
    q[0, :] = q[0, 0]
    sk[:] = sk[0]
    sv[:] = sv[0]
    o, _ = oracle_decode_beam(q, pk, pv, [5], sk, sv, [2, 2, 2, 2], g=1, scale=1.0)
    for w in range(1, 4):
        np.testing.assert_array_equal(o[0, w], o[0, 0])


def test_beam_with_empty_suffix_or_prefix_is_plain_decode():
    """No suffix rows: decode over the prefix; no prefix rows: decode over the suffix."""
    rng = np.random.default_rng(72)
    q, pk, pv, sk, sv = _beam_problem(rng, 2, 2, 4, 1, 3, 7, 5)
    o, lse = oracle_decode_beam(q, pk, pv, [7, 3], sk, sv, [0, 0, 0, 0], g=1, scale=1.0)
    od, lsed = oracle_decode(q.reshape(4, 4, 3), np.repeat(pk, 2, axis=0), np.repeat(pv, 2, axis=0),
                             [7, 7, 3, 3], g=1, scale=1.0)
    np.testing.assert_allclose(o.reshape(4, 4, 3), od, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse.reshape(4, 4), lsed, rtol=0, atol=1e-14)
    o, _ = oracle_decode_beam(q, pk, pv, [0, 0], sk, sv, [5, 1, 2, 3], g=1, scale=1.0)
    od, _ = oracle_decode(q.reshape(4, 4, 3), sk, sv, [5, 1, 2, 3], g=1, scale=1.0)
    np.testing.assert_allclose(o.reshape(4, 4, 3), od, rtol=0, atol=1e-15)
