"""GPU parity on the method's edge cases and on complete full-size tiles.

- exact ties of router logits (duplicated router rows, bias 0; an all-zero
  router): ids and their order must equal the oracle's bit for bit, equal
  logits going to the lower expert id;
- weight groups whose codes and fp16 scale are all zero (the quantiser's
  absmax = 0 case), in a selected routed expert and in the shared expert;
- the worst case for cancellation inside a group sum: constant positive
  tokens against codes that nearly cancel (+7 / -7 with a sum of -1 per group);
- at full size, every output element of all 32 tokens of a Zipf-routed decode
  batch, and of every token of the hottest expert's first complete 128-token
  tile of a 2048-token prefill.

The measured errors are printed (pytest -s shows them).
"""
import numpy as np
import pytest

import oracle
import synth
from tests import cases

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

FP32_TOL = 1e-3   # max |y - y_ref| <= FP32_TOL * max |y_ref|
BF16_TOL = 5e-3   # ||y - y_ref||_2 <= BF16_TOL * ||y_ref||_2


@pytest.fixture(scope="module")
def coli():
    import int4_expert_ffn_router_b200 as m
    return m


def _max_rel(y, y_ref):
    return float(np.abs(y - y_ref).max() / np.abs(y_ref).max())


def _layer(coli, c, wr, experts, bias=None, max_tokens=64):
    E, S = c["E"], c["S"]
    q = np.concatenate([e[0] for e in experts])
    s = np.concatenate([e[1] for e in experts])
    nq, ns = synth.expert_sizes(c["H"], c["I"])
    cfg = coli.make_config(c["H"], c["I"], E, c["K"], S, max_tokens)
    return coli.Layer(cfg, wr, bias, q[:E * nq], s[:E * ns], q[E * nq:] if S else None, s[E * ns:] if S else None,
                      device=0)


def _run(layer, x, gpu, mode):
    layer.set_fused(mode)
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.full_like(xd, float("nan"))
    layer.forward(xd, yd)
    layer.sync()
    return yd.cpu().numpy().astype(np.float64), layer.plan(x.shape[0])


# ---------------------------------------------------------------------- ties


@pytest.mark.parametrize("mode,T", [(1, 64), (1, 3), (0, 64), (1, 4)])
def test_router_ties_go_to_the_lower_id(gpu, coli, mode, T):
    """Rows 5 = row 3 (x10 of a base row) and rows 9 = row 7 (x5): their
    logits are bit-identical for every token, so slots decided between them
    are decided by the tie rule alone."""
    c = dict(cases.TINY, K=3)
    L = cases.host_layer(c, seed=21)
    wr = L["wr"].copy()
    base = wr[0].copy()
    wr[3] = wr[5] = (base * np.float32(10.0)).astype(np.float32)
    wr[7] = wr[9] = (base * np.float32(5.0)).astype(np.float32)
    layer = _layer(coli, c, wr, L["experts"])
    x = synth.x_f32(21, 1, T, c["H"])
    y, plan = _run(layer, x, gpu, mode)
    y_ref, ids_ref, w_ref = oracle.moe_forward(cases.oracle_cfg(c), wr, None, L["experts"], x)
    np.testing.assert_array_equal(plan["ids"], ids_ref)
    np.testing.assert_allclose(plan["weights"], w_ref, rtol=0, atol=1e-6)
    # the tie rule decided something: some token has both 3 and 5 (3 first), or 7 without 9
    rows = [list(r) for r in ids_ref]
    assert any(r[:2] == [3, 5] for r in rows)
    assert any(7 in r and 9 not in r for r in rows)
    err = _max_rel(y, y_ref)
    print(f"ties mode {mode} T={T}: max rel err {err:.2e}")
    assert err <= FP32_TOL
    layer.close()


@pytest.mark.parametrize("mode", [1, 0])
def test_all_zero_router_selects_the_lowest_ids(gpu, coli, mode):
    c = dict(cases.TINY, K=3)
    L = cases.host_layer(c, seed=22)
    wr = np.zeros_like(L["wr"])
    layer = _layer(coli, c, wr, L["experts"])
    x = synth.x_f32(22, 0, 5, c["H"])
    y, plan = _run(layer, x, gpu, mode)
    assert plan["ids"].tolist() == [[0, 1, 2]] * 5
    np.testing.assert_allclose(plan["weights"], 1.0 / 3.0, rtol=0, atol=1e-7)
    y_ref, ids_ref, _ = oracle.moe_forward(cases.oracle_cfg(c), wr, None, L["experts"], x)
    assert _max_rel(y, y_ref) <= FP32_TOL
    layer.close()


# ------------------------------------------------------------ zero-scale group


def _zero_groups(expert, H, I, rows_cols):
    """Zero the codes and the scale of the given (matrix, row, group) groups."""
    q, s = expert[0].copy(), expert[1].copy()
    nq_m, ns_m = I * H // 2, I * H // 64
    for m, r, g in rows_cols:
        cols = H if m < 2 else I
        qoff = m * nq_m + r * cols // 2 + g * 32
        soff = m * ns_m + r * cols // 64 + g
        q[qoff:qoff + 32] = 0
        s[soff] = 0
    return q, s


@pytest.mark.parametrize("mode,T", [(1, 1), (1, 4), (1, 13), (0, 13)])
def test_zero_scale_groups_in_routed_and_shared_experts(gpu, coli, mode, T):
    c = cases.TINY
    H, I, E = c["H"], c["I"], c["E"]
    L = cases.host_layer(c, seed=23)
    x = synth.x_f32(23, T, T, H)
    ids, _ = oracle.topk(oracle.router_logits(L["wr"], None, x), c["K"])
    experts = list(L["experts"])
    zero = [(0, 0, 0), (0, 5, 3), (1, 5, 3), (1, 200, 7), (2, 0, 0), (2, 100, 2), (2, 511, 3)]
    for e in {int(ids[0, 0]), E}:  # a selected routed expert and the shared expert
        experts[e] = _zero_groups(experts[e], H, I, zero)
    layer = _layer(coli, c, L["wr"], experts)
    y, plan = _run(layer, x, gpu, mode)
    y_ref, ids_ref, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, experts, x)
    np.testing.assert_array_equal(plan["ids"], ids_ref)
    err = _max_rel(y, y_ref)
    print(f"zero-scale groups mode {mode} T={T}: max rel err {err:.2e}")
    assert err <= FP32_TOL
    layer.close()


# ------------------------------------------------------- cancellation in a group


def _cancelling_expert(H, I, scale=2.0 ** -7):
    """Codes +7, -7, +7, ... in every group except the first input, +6: every
    group sums to -1, so each group sum is a small remainder of large terms."""
    def codes(rows, cols):
        q = np.where(np.arange(cols) % 2 == 0, 7, -7)[None, :].repeat(rows, 0)
        q[:, ::64] = 6
        return q
    return cases.expert_from_codes(codes(I, H), codes(I, H), codes(H, I), np.full((I, H // 64), scale),
                                   np.full((I, H // 64), scale), np.full((H, I // 64), scale))


@pytest.mark.parametrize("mode", [1, 0])
@pytest.mark.parametrize("T", [1, 2, 3, 4, 8])
def test_constant_positive_tokens_against_cancelling_codes(gpu, coli, mode, T):
    c = cases.TINY
    H, I, E = c["H"], c["I"], c["E"]
    L = cases.host_layer(c, seed=24)
    experts = [_cancelling_expert(H, I)] * (E + 1)
    # every element of token t equals 3 * (t + 1): every group's input sum is large
    x = np.repeat((3.0 * np.arange(1, T + 1, dtype=np.float32))[:, None], H, axis=1).astype(np.float32)
    layer = _layer(coli, c, L["wr"], experts)
    y, plan = _run(layer, x, gpu, mode)
    y_ref, ids_ref, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, experts, x)
    np.testing.assert_array_equal(plan["ids"], ids_ref)
    err = _max_rel(y, y_ref)
    print(f"cancelling codes mode {mode} T={T}: max rel err {err:.2e}")
    assert np.abs(y_ref).max() > 0
    assert err <= FP32_TOL
    layer.close()


# ---------------------------------------------------------- full-size tiles

_EXPERTS = {}


def _expert(e, H, I):
    if e not in _EXPERTS:
        _EXPERTS[e] = synth.expert(0, 0, e, H, I)
    return _EXPERTS[e]


def _oracle_rows(c, wr, bias, x):
    ids, _ = oracle.topk(oracle.router_logits(wr, bias, x), c["K"])
    experts = [None] * (c["E"] + c["S"])
    for e in set(ids.ravel().tolist()) | {c["E"] + j for j in range(c["S"])}:
        experts[e] = _expert(e, c["H"], c["I"])
    return oracle.moe_forward(cases.oracle_cfg(c), wr, bias, experts, x)[0]


def test_full_decode_batch32_every_output(gpu, coli):
    """All 32 tokens of a Zipf-routed full-size decode batch, element by element."""
    from tests import gpu_cases
    c = cases.FULL
    bias, _ = synth.zipf_bias(0, 0, c["E"])
    layer = gpu_cases.device_layer(c, seed=0, layer=0, bias=bias, max_tokens=32)
    x = synth.x_f32(2000, 0, 32, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    layer.sync()
    y = yd.cpu().numpy().astype(np.float64)
    layer.close()
    wr = synth.router(0, 0, c["E"], c["H"])
    y_ref = _oracle_rows(c, wr, bias, x)
    err = _max_rel(y, y_ref)
    per_token = np.abs(y - y_ref).max(axis=1) / np.abs(y_ref).max(axis=1)
    print(f"decode b32 full size: max rel err {err:.2e} (worst token {per_token.max():.2e})")
    assert err <= FP32_TOL


def test_full_prefill_2048_complete_tile_of_the_hottest_expert(gpu, coli):
    """Every token of the hottest expert's first complete 128-token tile, all
    of their output elements, within the bf16 tolerance token by token."""
    from tests import gpu_cases
    c = cases.FULL
    bias, _ = synth.zipf_bias(0, 0, c["E"])
    layer = gpu_cases.device_layer(c, seed=0, layer=0, bias=bias, max_tokens=2048)
    T = 2048
    xb = synth.x_bf16(3000, 0, T, c["H"])
    xd = torch.from_numpy(xb.view(np.int16)).to(gpu).view(torch.bfloat16)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    layer.sync()
    plan = layer.plan(T)
    yb = yd.view(torch.int16).cpu().numpy().view(np.uint16)
    layer.close()
    hot = int(np.argmax(plan["cnt"]))
    assert plan["cnt"][hot] >= 128
    toks = plan["tok"][plan["off"][hot]:plan["off"][hot] + 128]  # its first tile, in position order
    wr = synth.router(0, 0, c["E"], c["H"])
    y_ref = _oracle_rows(c, wr, bias, xb[toks])
    y = (yb[toks].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rel = np.linalg.norm(y - y_ref, axis=1) / np.linalg.norm(y_ref, axis=1)
    print(f"prefill 2048, expert {hot} ({plan['cnt'][hot]} tokens), first tile: worst token rel L2 {rel.max():.2e}")
    assert rel.max() <= BF16_TOL
