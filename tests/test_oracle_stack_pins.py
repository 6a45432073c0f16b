"""Pins for two oracle functions the GPU parity tests lean on, each against
something other than the oracle itself:

- the forced-routing path of the layer (a routing set made elsewhere, used
  for near-tie tokens): its weights are the softmax over the forced set's own
  logits, renormalised over that set;
- the stack of layers (the pages' model runs 48 MoE layers in a row, Strata
  tuning page, section 2 model table): r_0 = x, r_{l+1} = r_l +
  layer_l(bf16(RMSNorm(r_l))), the residual in fp64.
"""
import math

import numpy as np
import scipy.special

import oracle
from gen import MoeConfig, make_expert, make_layer, make_router, make_x


def _xf(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _small(H=64, I=32, E=8, k=3, T=6, seed=5):
    cfg = MoeConfig("t", H, I, E, k, T, "zipf")
    Wr, b = make_router(cfg, seed=seed)
    experts = np.stack([make_expert(H, I, seed, 0, e) for e in range(E)])
    shared = make_expert(H, I, seed, 0, E)
    return cfg, make_x(T, H, seed=seed), Wr, b, experts, shared


# ----------------------------------------------------------------------------
# forced routing (the layer's weights for a set chosen elsewhere)


def test_forced_set_equal_to_own_selection_is_bit_identical():
    cfg, x, Wr, b, experts, shared = _small()
    y, idx, w, gap = oracle.layer(x, Wr, b, experts, shared, cfg.top_k, cfg.inter)
    y2, idx2, w2, gap2 = oracle.layer(x, Wr, b, experts, shared, cfg.top_k, cfg.inter, forced_idx=idx)
    assert np.array_equal(idx2, idx) and np.array_equal(w2, w) and np.array_equal(y2, y)
    assert np.array_equal(gap2, gap)  # the gap always describes the oracle's own ranking


def test_forced_set_permuted_gives_permuted_weights():
    cfg, x, Wr, b, experts, shared = _small()
    y, idx, w, _ = oracle.layer(x, Wr, b, experts, shared, cfg.top_k, cfg.inter)
    perm = np.array([2, 0, 1])
    y2, idx2, w2, _ = oracle.layer(x, Wr, b, experts, shared, cfg.top_k, cfg.inter, forced_idx=idx[:, perm])
    assert np.array_equal(idx2, idx[:, perm])
    assert np.allclose(w2, w[:, perm], rtol=1e-15, atol=0)
    assert np.allclose(y2, y, rtol=0, atol=1e-14 * np.max(np.abs(y)))


def test_forced_set_weights_are_softmax_over_that_set():
    # A unit router (row e = unit vector at column p[e]) gives logits x[p[e]] + b[e] in closed form.  Forcing
    # the k LOWEST-logit experts must weight them by scipy's softmax over their own logits (a weight computed
    # over the free top-k set, or renormalised by its sum, fails), and y must be the shared expert plus that
    # weighted sum of the pinned single-expert FFN.
    H, I, E, k, T = 64, 32, 16, 3, 5
    rng = np.random.default_rng(9)
    p = rng.permutation(H)[:E]
    Wr = np.zeros((E, H), dtype=np.float32)
    Wr[np.arange(E), p] = 1.0
    b = rng.standard_normal(E).astype(np.float32)
    experts = np.stack([make_expert(H, I, 9, 0, e) for e in range(E)])
    shared = make_expert(H, I, 9, 0, E)
    x = make_x(T, H, seed=9)
    xv = _xf(x)
    logits = xv[:, p] + b.astype(np.float64)[None, :]
    forced = np.argsort(logits, axis=1, kind="stable")[:, :k].astype(np.int32)  # bottom-k
    y, idx, w, _ = oracle.layer(x, Wr, b, experts, shared, k, I, forced_idx=forced)
    want_w = scipy.special.softmax(np.take_along_axis(logits, forced.astype(np.int64), axis=1), axis=1)
    assert np.array_equal(idx, forced)
    assert np.allclose(w, want_w, rtol=1e-13, atol=0)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    for t in range(T):
        want_y = oracle.expert_forward(H, I, shared, xv[t])
        for j in range(k):
            want_y = want_y + want_w[t, j] * oracle.expert_forward(H, I, experts[forced[t, j]], xv[t])
        assert np.allclose(y[t], want_y, rtol=0, atol=1e-13 * np.max(np.abs(want_y)))


# ----------------------------------------------------------------------------
# the stack of layers


def _layers(cfg, L, seed=0):
    return [make_layer(cfg, seed=seed, layer=l) for l in range(L)]


def test_stack_zero_layers_is_the_input():
    cfg = MoeConfig("t", 64, 32, 8, 2, 4)
    x = make_x(4, 64, seed=1)
    r, idx, gap, nf, nm = oracle.stack(x, [], 2, 32)
    assert np.array_equal(r, _xf(x)) and idx.shape == (0, 4, 2) and nf == 0 and nm == 0


def test_stack_one_layer_is_residual_plus_layer_of_normalised_input():
    cfg = MoeConfig("t", 128, 64, 16, 4, 7, "zipf")
    lay = _layers(cfg, 1, seed=3)
    x = make_x(7, 128, seed=3)
    r, idx, gap, _, _ = oracle.stack(x, lay, 4, 64, eps=1e-6)
    u = oracle.double_to_bf16(oracle.rmsnorm(_xf(x), 1e-6))
    y, idx1, _, gap1 = oracle.layer(u, lay[0]["router_w"], lay[0]["router_b"], lay[0]["experts"], lay[0]["shared"],
                                    4, 64)
    assert np.array_equal(r, _xf(x) + y)
    assert np.array_equal(idx[0], idx1) and np.array_equal(gap[0], gap1)


def test_stack_composition_matches_layer_by_layer_loop():
    # Three different layers in order; a wrong layer order, a misplaced residual or normalisation fails.
    cfg = MoeConfig("t", 128, 64, 16, 4, 5, "zipf")
    lay = _layers(cfg, 3, seed=4)
    x = make_x(5, 128, seed=4)
    r, idx, _, _, _ = oracle.stack(x, lay, 4, 64)
    want = _xf(x)
    for l in range(3):
        u = oracle.double_to_bf16(oracle.rmsnorm(want, 1e-6))
        y, il, _, _ = oracle.layer(u, lay[l]["router_w"], lay[l]["router_b"], lay[l]["experts"], lay[l]["shared"], 4,
                                   64)
        assert np.array_equal(idx[l], il)
        want = want + y
    assert np.array_equal(r, want)
    r_rev, _, _, _, _ = oracle.stack(x, lay[::-1], 4, 64)
    assert not np.array_equal(r_rev, r)


def test_stack_of_zero_experts_leaves_the_residual_unchanged():
    cfg = MoeConfig("t", 64, 32, 8, 2, 4, "zipf")
    lay = _layers(cfg, 4, seed=2)
    for l in lay:
        for key in ("experts", "shared"):
            a = np.array(l[key]).reshape(-1, 10)
            a[:, 2:] = 0x55  # every code 1: w = d * (1 - 1) = 0
            l[key] = a.reshape(np.shape(l[key]))
    x = make_x(4, 64, seed=2)
    r, _, _, _, _ = oracle.stack(x, lay, 2, 32)
    assert np.array_equal(r, _xf(x))


def _diag_matrix(n, d_bits):
    """[n x n] Q2 matrix with d on the diagonal (code 2) and zero elsewhere (code 1), n == 32."""
    assert n == 32
    out = np.zeros((n, 10), dtype=np.uint8)
    for r in range(n):
        out[r, 0], out[r, 1] = d_bits & 0xFF, d_bits >> 8
        codes = np.ones(32, dtype=np.uint8)
        codes[r] = 2
        for j in range(32):
            out[r, 2 + (j >> 2)] |= codes[j] << (2 * (j & 3))
    return out.reshape(-1)


def test_stack_closed_form_diagonal_shared_expert():
    # H = I = 32; routed experts all zero; the shared expert's gate, up and down are diagonal with scales 1, 1/2
    # and 1/4, so each layer adds y_i = 1/4 * silu(u_i) * (1/2 * u_i) elementwise, u = bf16(RMSNorm(r)).
    H = I = 32
    f16 = lambda v: int(np.array([v], dtype=np.float16).view(np.uint16)[0])  # noqa: E731
    shared = np.concatenate([_diag_matrix(32, f16(1.0)), _diag_matrix(32, f16(0.5)), _diag_matrix(32, f16(0.25))])
    zero = shared.copy().reshape(-1, 10)
    zero[:, 2:] = 0x55
    E, k, L, T = 2, 1, 5, 6
    lay = [{"router_w": np.zeros((E, H), np.float32), "router_b": None,
            "experts": np.stack([zero.reshape(-1)] * E), "shared": shared} for _ in range(L)]
    x = make_x(T, H, seed=6)
    r, idx, gap, _, _ = oracle.stack(x, lay, k, I, eps=1e-6)
    want = _xf(x)
    for _ in range(L):
        v = want / np.sqrt(np.mean(want * want, axis=1, keepdims=True) + 1e-6)
        u = _xf(oracle.double_to_bf16(v))
        want = want + 0.25 * (u / (1.0 + np.exp(-u))) * (0.5 * u)
    assert np.allclose(r, want, rtol=1e-13, atol=1e-13)
    assert np.all(idx == 0) and np.all(gap == 0.0)  # all logits tie: the lower index, gap 0


def test_stack_follows_an_outside_routing_only_at_near_ties():
    cfg = MoeConfig("t", 64, 32, 8, 2, 4, "zipf")
    lay = _layers(cfg, 3, seed=8)
    x = make_x(4, 64, seed=8)
    r0, idx0, gap0, nf, nm = oracle.stack(x, lay, 2, 32)
    assert nf == 0 and nm == 0
    # the oracle's own routing, followed: nothing changes
    r1, idx1, _, nf, nm = oracle.stack(x, lay, 2, 32, follow_idx=idx0)
    assert np.array_equal(r1, r0) and np.array_equal(idx1, idx0) and nf == 0 and nm == 0
    # a different set with clear gaps is counted as a mismatch and not taken
    other = np.where(idx0 == 0, 1, 0).astype(np.int32)
    other[..., 1] = np.where(idx0[..., 0] == 7, 6, 7)
    r2, idx2, _, nf, nm = oracle.stack(x, lay, 2, 32, follow_idx=other, tie_gap=0.0)
    assert nf == 0 and nm == 3 * 4 and np.array_equal(r2, r0)
    # with every gap below the threshold the outside set is taken at every (layer, token) whose set differs
    r3, idx3, _, nf, nm = oracle.stack(x, lay, 2, 32, follow_idx=other, tie_gap=math.inf)
    assert nf == 3 * 4 and nm == 0 and np.array_equal(idx3, other)
    assert not np.array_equal(r3, r0)


def test_stack_in_chunks_of_layers_equals_one_call():
    cfg = MoeConfig("t", 64, 32, 8, 2, 4, "zipf")
    lay = _layers(cfg, 5, seed=12)
    x = make_x(4, 64, seed=12)
    r, idx, gap, _, _ = oracle.stack(x, lay, 2, 32)
    r2, idx2, gap2, _, _ = oracle.stack(x, lay[:2], 2, 32)
    r3, idx3, gap3, _, _ = oracle.stack(x, lay[2:], 2, 32, resid_in=r2)
    assert np.array_equal(r3, r) and np.array_equal(np.concatenate([idx2, idx3]), idx)
    assert np.array_equal(np.concatenate([gap2, gap3]), gap)
