"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Every check here is independent of the oracle's own formulas: closed forms,
library routines on special cases, invariants, and brute force on tiny inputs.
A plausible slip anywhere in the oracle (a dropped term, a wrong sign, a
transposed operand, gate/up swapped, a lost shared expert, a wrong tie rule)
fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from tests import cases

# --------------------------------------------------------------------- decoding


def test_f16_decode_matches_numpy_on_all_finite_patterns():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(ref)
    got = np.array([oracle.f16(int(b)) for b in bits[finite][::7]])
    np.testing.assert_array_equal(got, ref[finite][::7])
    # the few landmarks exactly
    assert oracle.f16(0x3C00) == 1.0
    assert oracle.f16(0xC000) == -2.0
    assert oracle.f16(0x7BFF) == 65504.0
    assert oracle.f16(0x0001) == 2.0 ** -24
    assert oracle.f16(0x0400) == 2.0 ** -14
    assert math.isinf(oracle.f16(0x7C00))


def test_bf16_decode():
    assert oracle.bf16(0x3F80) == 1.0
    assert oracle.bf16(0xC040) == -3.0
    assert oracle.bf16(0x0001) == 2.0 ** -133
    v = np.float32(-1.2345678e-3)
    b = int(np.array([v]).view(np.uint32)[0] >> 16)
    assert oracle.bf16(b) == float(np.array([b << 16], np.uint32).view(np.float32)[0])


def test_nibble_decode_handcrafted():
    # 0x8F: low nibble 0xF -> -1 (element 0), high nibble 0x8 -> -8 (element 1)
    # 0x70: low 0 (element 2), high 7 (element 3)
    row = np.array([0x8F, 0x70, 0x21, 0xE9], np.uint8)
    assert [oracle.code(row, c) for c in range(8)] == [-1, -8, 0, 7, 1, 2, -7, -2]


def test_dequant_handcrafted_group_scales():
    codes = np.array([[(c % 16) - 8 for c in range(128)]], np.int64)
    q = cases.pack_codes(codes)
    s = cases.f16_bits([[0.5, -0.25]])
    w = oracle.dequant(q, s, 1, 128)
    expect = np.concatenate([codes[0, :64] * 0.5, codes[0, 64:] * -0.25])
    np.testing.assert_array_equal(w[0], expect)


@pytest.mark.parametrize("matrix,rows,cols", [(synth.GATE, 256, 512), (synth.UP, 256, 512), (synth.DOWN, 512, 256)])
def test_int4_gs64_round_trip_within_half_step(matrix, rows, cols):
    """Encoding then decoding moves every weight by at most half a step s/2
    (int4 gs64 container); codes stay in [-8, 7]; the scale is absmax/7 in fp16."""
    H, I = 512, 256
    q, s = synth.expert(3, 0, 5, H, I)
    nq, ns = H * I // 2, H * I // 64
    qm = q[matrix * nq:(matrix + 1) * nq]
    sm = s[matrix * ns:(matrix + 1) * ns]
    w = synth.matrix_f32(3, 0, 5, matrix, rows, cols).astype(np.float64)
    wd = oracle.dequant(qm, sm, rows, cols)
    sc = np.repeat(sm.view(np.float16).astype(np.float64).reshape(rows, cols // 64), 64, axis=1)
    assert np.all(np.abs(w - wd) <= sc / 2 + 0.0)
    # the scale rule, through numpy's own fp16 rounding
    amax = np.abs(w.reshape(rows, cols // 64, 64)).max(axis=2).astype(np.float32)
    np.testing.assert_array_equal(sm.reshape(rows, cols // 64), (amax / np.float32(7)).astype(np.float16).view(np.uint16))
    codes = np.rint(wd / np.where(sc == 0, 1, sc))
    assert codes.min() >= -8 and codes.max() <= 7


# ----------------------------------------------------------------------- router


def test_router_logits_are_a_matmul_plus_bias():
    rng = np.random.default_rng(1)
    wr = rng.standard_normal((16, 128)).astype(np.float32)
    x = rng.standard_normal((5, 128)).astype(np.float32)
    b = rng.standard_normal(16).astype(np.float32)
    got = oracle.router_logits(wr, b, x)
    ref = x.astype(np.float64) @ wr.astype(np.float64).T + b.astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # bf16 activations are widened exactly
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    xw = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    np.testing.assert_allclose(oracle.router_logits(wr, None, xb), xw @ wr.astype(np.float64).T, rtol=0, atol=1e-12)


def test_topk_brute_force_and_exactly_k_distinct():
    rng = np.random.default_rng(2)
    T, E, K = 64, 256, 8
    logits = rng.standard_normal((T, E))
    ids, w = oracle.topk(logits, K)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-logits[t, e], e))
        assert list(ids[t]) == order[:K]
        assert len(set(ids[t])) == K
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)


def test_topk_ties_go_to_lower_id_and_k_equals_e():
    logits = np.zeros((2, 6))
    logits[1] = [1.0, 3.0, 3.0, 0.5, 3.0, -1.0]
    ids, w = oracle.topk(logits, 3)
    assert list(ids[0]) == [0, 1, 2]
    assert list(ids[1]) == [1, 2, 4]
    np.testing.assert_allclose(w, 1.0 / 3.0, rtol=0, atol=1e-16)
    ids, _ = oracle.topk(logits, 6)
    assert sorted(ids[0]) == list(range(6)) and list(ids[1]) == [1, 2, 4, 0, 3, 5]


def test_topk_weights_closed_form_and_full_softmax_form():
    # logits ln 1, ln 2, ln 3, ln 4 -> top-2 picks ids 3, 2 with weights 4/7, 3/7
    logits = np.log(np.array([[1.0, 2.0, 3.0, 4.0]]))
    ids, w = oracle.topk(logits, 2)
    assert list(ids[0]) == [3, 2]
    np.testing.assert_allclose(w[0], [4 / 7, 3 / 7], rtol=0, atol=1e-15)
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((32, 256)) * 3
    ids, w = oracle.topk(lg, 8)
    np.testing.assert_allclose(oracle.weights_full_softmax(lg, ids), w, rtol=0, atol=1e-15)


@pytest.mark.parametrize("p,ids_ref,w_ref", [
    (0.65, [3, 2, -1, -1], [4 / 7, 3 / 7, 0, 0]),   # 0.4 < 0.65 <= 0.7
    (0.75, [3, 2, 1, -1], [4 / 9, 3 / 9, 2 / 9, 0]),  # 0.7 < 0.75 <= 0.9
    (0.3, [3, -1, -1, -1], [1, 0, 0, 0]),            # the first expert alone reaches p
    (0.95, [3, 2, 1, 0], [0.4, 0.3, 0.2, 0.1]),      # all four needed
    (1.0, [3, 2, 1, 0], [0.4, 0.3, 0.2, 0.1]),       # p = 1: plain top-K
])
def test_expert_top_p_closed_forms(p, ids_ref, w_ref):
    """Adaptive expert top-p on logits ln 1..ln 4 (K = 4, weights 0.4, 0.3,
    0.2, 0.1): keep the shortest prefix whose weights reach p, renormalise."""
    logits = np.log(np.array([[1.0, 2.0, 3.0, 4.0]]))
    ids, w = oracle.topk(logits, 4, top_p=p)
    assert ids[0].tolist() == ids_ref
    np.testing.assert_allclose(w[0], w_ref, rtol=0, atol=1e-15)


def test_expert_top_p_invariants_on_random_routers():
    """Kept counts grow with p, kept weights sum to 1, the kept ids are the
    plain top-K's prefix, and the mass the kept experts carried before the
    renormalisation reaches p while the prefix one shorter does not."""
    rng = np.random.default_rng(11)
    lg = rng.standard_normal((200, 64)) * 2
    ids0, w0 = oracle.topk(lg, 8)
    prev = None
    for p in (0.2, 0.5, 0.7, 0.9, 0.99):
        ids, w = oracle.topk(lg, 8, top_p=p)
        keep = (ids >= 0).sum(axis=1)
        assert keep.min() >= 1
        if prev is not None:
            assert (keep >= prev).all()
        prev = keep
        for t in range(200):
            n = keep[t]
            assert ids[t, :n].tolist() == ids0[t, :n].tolist() and (ids[t, n:] == -1).all()
            np.testing.assert_allclose(w[t, :n].sum(), 1.0, rtol=0, atol=1e-14)
            assert (w[t, n:] == 0).all()
            assert w0[t, :n].sum() >= p - 1e-15
            assert n == 1 or w0[t, :n - 1].sum() < p + 1e-15
            np.testing.assert_allclose(w[t, :n], w0[t, :n] / w0[t, :n].sum(), rtol=1e-15, atol=0)


def test_expert_top_p_layer_reductions(tiny):
    """A layer with top-K and p below every token's top weight is the top-1
    layer (one expert at weight 1); p = 1 is the plain layer; in between the
    output equals the layer rebuilt from single-expert calls over the kept
    experts with the renormalised weights."""
    c, L, x = tiny
    cK = dict(c, K=4)
    y1, ids1, _ = oracle.moe_forward(cases.oracle_cfg(dict(c, K=1)), L["wr"], None, L["experts"], x)
    yp, idsp, wp = oracle.moe_forward(cases.oracle_cfg(cK, top_p=1e-9), L["wr"], None, L["experts"], x)
    assert (idsp[:, 1:] == -1).all() and (idsp[:, 0] == ids1[:, 0]).all() and (wp[:, 0] == 1.0).all()
    np.testing.assert_array_equal(yp, y1)
    yK, idsK, _ = oracle.moe_forward(cases.oracle_cfg(cK), L["wr"], None, L["experts"], x)
    y_one, ids_one, _ = oracle.moe_forward(cases.oracle_cfg(cK, top_p=1.0), L["wr"], None, L["experts"], x)
    np.testing.assert_array_equal(yK, y_one)
    y7, ids7, w7 = oracle.moe_forward(cases.oracle_cfg(cK, top_p=0.7), L["wr"], None, L["experts"], x)
    logits = oracle.router_logits(L["wr"], None, x)
    ids_k, w_k = oracle.topk(logits, 4)
    assert (ids7 >= 0).sum() < ids7.size            # something was dropped
    for t in range(c["T"]):
        xt = x[t].astype(np.float64)
        n = int((ids7[t] >= 0).sum())
        ref = oracle.expert_ffn(*L["experts"][c["E"]], c["H"], c["I"], xt)
        for k in range(n):
            ref = ref + (w_k[t, k] / w_k[t, :n].sum()) * oracle.expert_ffn(*L["experts"][ids_k[t, k]], c["H"], c["I"], xt)
        np.testing.assert_allclose(y7[t], ref, rtol=0, atol=1e-13 * np.abs(ref).max())


def test_topk_rejects_nan():
    with pytest.raises(ValueError):
        oracle.topk(np.array([[0.0, np.nan, 1.0]]), 2)


# ------------------------------------------------------------------------ union


def test_union_invariants_against_python_sets():
    rng = np.random.default_rng(4)
    T, K, E = 40, 8, 256
    ids = np.stack([rng.choice(E, K, replace=False, p=None) for _ in range(T)]).astype(np.int32)
    # skew: half the tokens share experts 0..7
    ids[::2] = np.arange(8)
    u = oracle.union(ids, E)
    assert int(u["cnt"].sum()) == T * K
    assert list(u["unique"]) == sorted(set(ids.ravel().tolist()))
    assert len(set(u["unique"].tolist())) == len(u["unique"])
    for e in range(E):
        toks = [t for t in range(T) for k in range(K) if ids[t, k] == e]
        assert u["cnt"][e] == len(toks)
        assert list(u["tok"][u["off"][e]:u["off"][e + 1]]) == toks  # ascending tokens
    for t in range(T):
        for k in range(K):
            p = u["pos"][t, k]
            assert u["tok"][p] == t and u["off"][ids[t, k]] <= p < u["off"][ids[t, k] + 1]
    assert sorted(u["pos"].ravel().tolist()) == list(range(T * K))  # a permutation


def test_union_touches_each_unique_expert_once_and_the_per_layer_fraction():
    """Batch 1, full-size shapes: 8 of 256 chosen; streamed parameters are the
    8 routed + 1 shared experts plus the router, 3.52% of the layer."""
    H, I, E, K = 6144, 2048, 256, 8
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((1, E))
    ids, _ = oracle.topk(logits, K)
    u = oracle.union(ids, E)
    assert len(u["unique"]) == 8
    per_expert = 3 * H * I
    touched = (len(u["unique"]) + 1) * per_expert + E * H
    total = (E + 1) * per_expert + E * H
    assert touched == 9 * 37_748_736 + 1_572_864
    assert abs(touched / total - 0.0352) < 5e-4
    # the pages' whole-model figure (40B of 744B, ~5.4%) from their own counts:
    # 75 layers x 8 routed experts + 17B dense part, over 19,456 experts + 17B
    whole = (75 * 8 * per_expert + 17e9) / (19456 * per_expert + 17e9)
    assert abs(whole - 0.054) < 0.002


# ----------------------------------------------------------------------- expert


def _basis_expert(H, I, j, gate_q, up_q, sg, su):
    """Gate/up have one nonzero column j; down is the identity on the first I rows."""
    G = np.zeros((I, H), np.int64)
    U = np.zeros((I, H), np.int64)
    G[:, j] = gate_q
    U[:, j] = up_q
    D = np.zeros((H, I), np.int64)
    D[np.arange(I), np.arange(I)] = 1
    return cases.expert_from_codes(G, U, D, np.full((I, H // 64), sg), np.full((I, H // 64), su),
                                   np.full((H, I // 64), 1.0))


def test_expert_ffn_closed_form_on_a_basis_vector():
    """x = a e_j: g_r = a G[r][j], u_r = a U[r][j], h_r = silu(g_r) u_r, and with
    D = [I; 0] the output is h followed by zeros. H != I catches transposes;
    distinct gate/up codes catch a gate/up swap."""
    H, I, j, a = 128, 64, 37, 1.5
    gate_q = np.array([(r % 15) - 7 for r in range(I)])
    up_q = np.array([7 - (r % 13) for r in range(I)])
    q, s = _basis_expert(H, I, j, gate_q, up_q, 0.5, 0.25)
    x = np.zeros(H)
    x[j] = a
    out, h = oracle.expert_ffn(q, s, H, I, x, want_h=True)
    for r in range(I):
        g = a * gate_q[r] * 0.5
        u = a * up_q[r] * 0.25
        hr = g / (1 + math.exp(-g)) * u
        assert h[r] == pytest.approx(hr, rel=1e-15, abs=1e-300)
        assert out[r] == pytest.approx(hr, rel=1e-15, abs=1e-300)
    assert np.all(out[I:] == 0.0)


def test_expert_ffn_silu_zero_and_dense_library_form():
    H, I = 128, 64
    q, s = synth.expert(7, 0, 0, H, I)
    assert np.all(oracle.expert_ffn(q, s, H, I, np.zeros(H)) == 0.0)
    # same expert through numpy's matmul on the decoded matrices
    nq, ns = H * I // 2, H * I // 64
    G = oracle.dequant(q[:nq], s[:ns], I, H)
    U = oracle.dequant(q[nq:2 * nq], s[ns:2 * ns], I, H)
    D = oracle.dequant(q[2 * nq:], s[2 * ns:], H, I)
    x = np.random.default_rng(6).standard_normal(H)
    g, u = G @ x, U @ x
    ref = D @ (g / (1 + np.exp(-g)) * u)
    np.testing.assert_allclose(oracle.expert_ffn(q, s, H, I, x), ref, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------------ layer


@pytest.fixture(scope="module")
def tiny():
    c = cases.TINY
    L = cases.host_layer(c, seed=c["seed"])
    x = synth.x_f32(c["seed"], 0, c["T"], c["H"])
    return c, L, x


def test_sparse_equals_dense_with_unselected_gates_zeroed(tiny):
    """Sparse selection is checked by forcing full selection against the dense
    computation (as the colibri pages validate their sparse attention)."""
    c, L, x = tiny
    cfg = cases.oracle_cfg(c)
    y, ids, w = oracle.moe_forward(cfg, L["wr"], L["bias"], L["experts"], x)
    yd = oracle.moe_forward(cfg, L["wr"], L["bias"], L["experts"], x, dense=True)
    np.testing.assert_allclose(y, yd, rtol=0, atol=1e-12 * np.abs(yd).max())
    assert ids.shape == (c["T"], c["K"]) and all(len(set(r)) == c["K"] for r in ids)


def test_layer_decomposes_into_shared_plus_weighted_routed(tiny):
    """y = shared(x) + sum_k w_k E_k(x): rebuilt from single-expert calls."""
    c, L, x = tiny
    cfg = cases.oracle_cfg(c)
    y, ids, w = oracle.moe_forward(cfg, L["wr"], L["bias"], L["experts"], x)
    logits = oracle.router_logits(L["wr"], None, x)
    ids2, w2 = oracle.topk(logits, c["K"])
    np.testing.assert_array_equal(ids, ids2)
    for t in range(c["T"]):
        xt = x[t].astype(np.float64)
        ref = oracle.expert_ffn(*L["experts"][c["E"]], c["H"], c["I"], xt)
        for k in range(c["K"]):
            ref = ref + w2[t, k] * oracle.expert_ffn(*L["experts"][ids[t, k]], c["H"], c["I"], xt)
        np.testing.assert_allclose(y[t], ref, rtol=0, atol=1e-13 * np.abs(ref).max())


def test_shared_only_when_routed_experts_are_zero(tiny):
    c, L, x = tiny
    cfg = cases.oracle_cfg(c)
    zero = (np.zeros_like(L["experts"][0][0]), np.zeros_like(L["experts"][0][1]))
    experts = [zero] * c["E"] + L["experts"][c["E"]:]
    y, _, _ = oracle.moe_forward(cfg, L["wr"], None, experts, x)
    for t in range(c["T"]):
        ref = oracle.expert_ffn(*L["experts"][c["E"]], c["H"], c["I"], x[t].astype(np.float64))
        np.testing.assert_array_equal(y[t], ref)


def test_bias_changes_selection_and_no_shared_expert():
    """A large bias on experts 3 and 9 forces them to be chosen (top-2); with no
    shared expert the output is exactly the two weighted routed experts."""
    c = dict(cases.TINY, S=0)
    L = cases.host_layer(c, seed=1)
    bias = np.zeros(c["E"], np.float32)
    bias[3], bias[9] = 50.0, 49.0
    x = synth.x_f32(1, 0, 2, c["H"])
    cfg = cases.oracle_cfg(c)
    y, ids, w = oracle.moe_forward(cfg, L["wr"], bias, L["experts"], x)
    assert ids.tolist() == [[3, 9], [3, 9]]
    for t in range(2):
        xt = x[t].astype(np.float64)
        ref = w[t, 0] * oracle.expert_ffn(*L["experts"][3], c["H"], c["I"], xt) + \
            w[t, 1] * oracle.expert_ffn(*L["experts"][9], c["H"], c["I"], xt)
        np.testing.assert_allclose(y[t], ref, rtol=0, atol=1e-13 * np.abs(ref).max())


def test_empty_batch():
    c = cases.TINY
    L = cases.host_layer(c, seed=0, which=[])
    y, ids, w = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], np.zeros((0, c["H"]), np.float32))
    assert y.shape == (0, c["H"])


def test_missing_selected_expert_is_an_error():
    c = cases.TINY
    L = cases.host_layer(c, seed=0, which=[c["E"]])
    with pytest.raises(ValueError):
        oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], synth.x_f32(0, 0, 1, c["H"]))


# ------------------------------------------------------------------------ stack


def test_rmsnorm_closed_forms():
    x = np.full((1, 64), -3.0)
    np.testing.assert_allclose(oracle.rmsnorm(x, eps=0.0), -1.0, rtol=1e-15)
    x = np.random.default_rng(7).standard_normal((3, 256)) * 5
    n = oracle.rmsnorm(x, eps=0.0)
    np.testing.assert_allclose((n ** 2).mean(axis=1), 1.0, rtol=1e-14)
    r = n / x
    np.testing.assert_allclose(r, np.broadcast_to(r[:, :1], r.shape), rtol=1e-14)  # one scale per token


def test_stack_step_is_residual_of_normalised_layer(tiny):
    c, L, x = tiny
    cfg = cases.oracle_cfg(c)
    x0 = (x * 7.0).astype(np.float32)
    xs = x0.copy()
    ids = oracle.stack_step(cfg, L["wr"], None, L["experts"], xs)
    nf = oracle.rmsnorm(x0.astype(np.float64)).astype(np.float32)
    y, ids2, _ = oracle.moe_forward(cfg, L["wr"], None, L["experts"], nf)
    np.testing.assert_array_equal(ids, ids2)
    np.testing.assert_array_equal(xs, (x0.astype(np.float64) + y).astype(np.float32))


def _zero_layer(c):
    """Zero router, all-zero routed and shared experts (codes 0, scales 0)."""
    nq, ns = synth.expert_sizes(c["H"], c["I"])
    zero = (np.zeros(nq, np.uint8), np.zeros(ns, np.uint16))
    return np.zeros((c["E"], c["H"]), np.float32), [zero] * (c["E"] + c["S"])


def test_stack_step_with_a_zero_layer_returns_x_bit_for_bit():
    """Zero router (all logits tie at 0) and all-zero experts: the MoE term is
    exactly 0, so the step must hand back x itself. Replacing x by the layer
    output, or scaling the residual, fails here."""
    c = cases.TINY
    wr, experts = _zero_layer(c)
    x = (synth.x_f32(9, 0, 3, c["H"]) * 13.0).astype(np.float32)
    xs = x.copy()
    ids = oracle.stack_step(cases.oracle_cfg(c), wr, None, experts, xs)
    assert np.array_equal(xs.view(np.uint32), x.view(np.uint32))
    assert ids.tolist() == [[0, 1]] * 3  # equal logits go to the lower ids


def test_stack_step_increment_does_not_depend_on_the_scale_of_x(tiny):
    """With eps = 0, RMSNorm(2^k x) == RMSNorm(x) exactly (every operation is
    scaled by a power of two), so the increment x_out - x of a step must be the
    same for x and 2^k x up to the final fp32 rounding of each sum. A norm
    applied to the layer output instead of its input, or a missing norm, makes
    the increment grow with the scale (SwiGLU is not homogeneous)."""
    c, L, x = tiny
    cfg = cases.oracle_cfg(c)
    x0 = x.astype(np.float32)
    inc = {}
    out = {}
    for k in (0, 5):
        xs = (x0 * np.float32(2.0 ** k)).astype(np.float32)
        xin = xs.astype(np.float64)
        oracle.stack_step(cfg, L["wr"], None, L["experts"], xs, eps=0.0)
        out[k] = xs
        inc[k] = xs.astype(np.float64) - xin
    half_ulp = lambda a: np.spacing(np.abs(a).astype(np.float32)).astype(np.float64) / 2
    bound = half_ulp(out[0]) + half_ulp(out[5])
    assert np.all(np.abs(inc[5] - inc[0]) <= bound)
    assert np.abs(inc[0]).max() > 1e-3  # the layer term is not trivially zero


def test_stack_step_closed_form_with_one_basis_expert():
    """Zero router and routed experts; the shared expert has gate/up codes only
    in column j and down = identity on the first I rows. Then, with
    n = x / sqrt(mean(x^2) + eps) rounded to fp32,
        out[r] = fp32(x[r] + silu(n_j G_rj sg) * (n_j U_rj su))   for r < I,
        out[r] = x[r]                                             for r >= I.
    eps is large enough that putting it outside the square root, or using the
    sum instead of the mean, changes n_j by far more than the tolerance."""
    c = dict(cases.TINY, S=1)
    H, I, E = c["H"], c["I"], c["E"]
    j, eps = 37, 0.25
    gate_q = np.array([(r % 15) - 7 for r in range(I)])
    up_q = np.array([7 - (r % 13) for r in range(I)])
    wr, experts = _zero_layer(c)
    experts = list(experts)
    experts[E] = _basis_expert(H, I, j, gate_q, up_q, 0.5, 0.25)
    rng = np.random.default_rng(11)
    x = (rng.integers(-8, 9, size=(2, H)) * 0.125).astype(np.float32)  # sum of squares exact in fp64
    xs = x.copy()
    oracle.stack_step(cases.oracle_cfg(c), wr, None, experts, xs, eps=eps)
    for t in range(2):
        xt = x[t].astype(np.float64)
        ms = float(np.sum(xt * xt)) / H
        nj = float(np.float32(xt[j] / math.sqrt(ms + eps)))
        ref = xt.copy()
        for r in range(I):
            g = nj * gate_q[r] * 0.5
            u = nj * up_q[r] * 0.25
            ref[r] = xt[r] + g / (1.0 + math.exp(-g)) * u
        ref32 = ref.astype(np.float32).astype(np.float64)
        np.testing.assert_allclose(xs[t].astype(np.float64), ref32, rtol=2.5e-7, atol=1e-30)
        assert np.array_equal(xs[t, I:], x[t, I:])


# ------------------------------------------------------------- page figures


def _page_figures():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "page_figures.txt")
    out = {}
    with open(path, encoding="utf-8") as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                out[k] = float(v)
    return out


def test_expert_size_and_counts_match_the_pages_figures():
    """The full-size expert (hidden 6144, inter 2048, int4 gs64 with fp16
    scales) against the sizes the Colibrì background section prints: about
    19 MB per expert, 19,456 routed experts (75 layers x 256 + the MTP head)
    taking about 370 GB, and 6,300 of them filling 120 GB of VRAM."""
    fig = _page_figures()
    H, I = 6144, 2048
    per_expert = 3 * H * I // 2 + 3 * H * I // 64 * 2   # nibbles + fp16 scales
    assert per_expert == 20_054_016
    assert abs(per_expert / 1e6 - fig["expert_megabytes_int4"]) / fig["expert_megabytes_int4"] < 0.1
    assert fig["moe_layers"] * fig["routed_experts_per_layer"] + fig["routed_experts_per_layer"] == fig["routed_experts_total"]
    total_gb = fig["routed_experts_total"] * per_expert / 1e9
    assert abs(total_gb - fig["routed_experts_total_gigabytes"]) / fig["routed_experts_total_gigabytes"] < 0.1
    per_hot = fig["vram_hot_gigabytes"] * 1e9 / fig["vram_hot_experts"]
    assert abs(per_hot - per_expert) / per_expert < 0.1
    # 8 of the 256 experts per layer; the whole model's active share from these counts
    assert fig["routed_per_token"] == 8 and fig["routed_experts_per_layer"] == 256
    w = 3 * H * I
    whole = (fig["moe_layers"] * fig["routed_per_token"] * w + fig["dense_params_billion"] * 1e9) / \
            (fig["routed_experts_total"] * w + fig["dense_params_billion"] * 1e9)
    assert abs(whole - fig["active_fraction"]) < 0.002
    assert abs(fig["active_params_billion"] / fig["total_params_billion"] - fig["active_fraction"]) < 0.001
