"""Pins for the fp64 oracle: closed forms, invariants, special cases and brute
force, each independent of the oracle's own code.

The pages print no worked example for this layer (no sample block bytes, no
logits, no outputs), so every pin below comes from the formats' definitions,
the mathematics of the layer, or an independent library routine.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from gen import MoeConfig, make_expert, make_router, make_x, f32_to_bf16_bits

# ----------------------------------------------------------------------------
# scalar formats


def test_half_decode_hand_values():
    # IEEE 754 binary16 patterns whose values follow from the definition.
    table = {
        0x3C00: 1.0,
        0xC000: -2.0,
        0x7BFF: 65504.0,
        0x0001: 2.0 ** -24,
        0x03FF: 1023 * 2.0 ** -24,
        0x0400: 2.0 ** -14,
        0x3555: 0.333251953125,
        0x3800: 0.5,
        0x2E66: 0.0999755859375,
        0x0000: 0.0,
    }
    for bits, val in table.items():
        assert oracle.half_to_double(bits) == val, hex(bits)
    assert math.copysign(1.0, oracle.half_to_double(0x8000)) == -1.0
    assert oracle.half_to_double(0x7C00) == math.inf
    assert oracle.half_to_double(0xFC00) == -math.inf
    assert math.isnan(oracle.half_to_double(0x7E00))


def test_half_decode_all_patterns_match_numpy():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decode_all_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32)
    ref = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    got = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_double_to_bf16_round_to_nearest_even():
    # Values placed at known fractions between two adjacent bf16 numbers.
    rng = np.random.default_rng(5)
    base_bits = rng.integers(0x0080, 0x7F00, size=400).astype(np.uint32)  # positive normals
    lo = (base_bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    hi = ((base_bits + 1) << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    ulp = hi - lo
    for frac in (0.0, 0.25, 0.49, 0.5, 0.51, 0.75):
        v = lo + frac * ulp
        got = oracle.double_to_bf16(np.concatenate([v, -v])).astype(np.uint32)
        if frac < 0.5:
            want = base_bits
        elif frac > 0.5:
            want = base_bits + 1
        else:  # tie: to the even pattern
            want = np.where(base_bits % 2 == 0, base_bits, base_bits + 1)
        assert np.array_equal(got[:400], want)
        assert np.array_equal(got[400:], want | 0x8000)


# ----------------------------------------------------------------------------
# Q2 blocks


def _block(d_bits: int, codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    assert codes.size == 32
    blk = np.zeros(10, dtype=np.uint8)
    blk[0] = d_bits & 0xFF
    blk[1] = d_bits >> 8
    for j in range(32):
        blk[2 + (j >> 2)] |= (int(codes[j]) & 3) << (2 * (j & 3))
    return blk


@pytest.mark.parametrize("d_bits", [0x3C00, 0x2E66, 0x0001, 0x0400, 0x7BFF, 0xBC00, 0x0000, 0x1A3F])
def test_dequant_closed_form_table(d_bits):
    d = float(np.array([d_bits], dtype=np.uint16).view(np.float16)[0])
    hand = {0: -d, 1: 0.0, 2: d, 3: 2.0 * d}
    for q in range(4):
        w = oracle.dequant_block(_block(d_bits, [q] * 32))
        assert np.all(w == hand[q]), (hex(d_bits), q)


def test_dequant_element_order():
    # A single code 3 at position j with all others 1: only element j is nonzero (2d).
    for j in range(32):
        codes = [1] * 32
        codes[j] = 3
        w = oracle.dequant_block(_block(0x3C00, codes))
        want = np.zeros(32)
        want[j] = 2.0
        assert np.array_equal(w, want), j


def test_dequant_round_trip_bit_exact():
    # The pages' canonical check (devlabs page, section 4, second layer): Q2_0
    # re-encoded through the affine bias=-1 codebook is bit-exact, max|d| = 0.
    rng = np.random.default_rng(1)
    nblk = 5000
    d = np.abs(rng.standard_normal(nblk).astype(np.float32) * 0.02).astype(np.float16)
    d[d == 0] = np.float16(1e-3)
    qs = rng.integers(0, 256, size=(nblk, 8), dtype=np.uint8)
    blocks = np.concatenate([d.view(np.uint8).reshape(nblk, 2), qs], axis=1)
    W = oracle.dequant_matrix(blocks.reshape(-1), 1, nblk * 32).reshape(nblk, 32)
    dd = d.astype(np.float64)[:, None]
    q = np.rint(W / dd).astype(np.int64) + 1
    assert q.min() >= 0 and q.max() <= 3
    re = np.zeros((nblk, 8), dtype=np.uint8)
    for j in range(32):
        re[:, j >> 2] |= (q[:, j].astype(np.uint8) << (2 * (j & 3)))
    rebuilt = np.concatenate([np.float16(d).view(np.uint8).reshape(nblk, 2), re], axis=1)
    assert np.array_equal(rebuilt, blocks)
    assert np.max(np.abs(W - dd * (q - 1))) == 0.0


def np_dequant(blocks: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Independent vectorised decode of the canonical format (numpy float16)."""
    b = np.ascontiguousarray(blocks, dtype=np.uint8).reshape(rows, cols // 32, 10)
    d = np.ascontiguousarray(b[..., 0:2]).view(np.float16)[..., 0].astype(np.float64)
    qs = b[..., 2:10]
    q = np.stack([(qs >> (2 * s)) & 3 for s in range(4)], axis=-1).reshape(rows, cols // 32, 32)
    return (d[..., None] * (q.astype(np.float64) - 1.0)).reshape(rows, cols)


def test_dequant_matrix_matches_independent_decode():
    ex = make_expert(256, 128, seed=3, layer=0, expert=0)
    gate = ex[: 128 * 256 // 32 * 10]
    assert np.array_equal(oracle.dequant_matrix(gate, 128, 256), np_dequant(gate, 128, 256))


# ----------------------------------------------------------------------------
# routing


@pytest.mark.parametrize("E,k", [(4, 1), (4, 2), (4, 4), (16, 1), (16, 2), (16, 10), (16, 16), (512, 1), (512, 10),
                                 (512, 512)])
def test_topk_matches_full_stable_sort(E, k):
    rng = np.random.default_rng(E * 1000 + k)
    logits = rng.standard_normal((64, E))
    logits[::2] = np.round(logits[::2] * 4) / 4  # coarse grid: many exact ties
    logits[5] = 0.0                               # every logit tied
    idx, w, gap = oracle.topk(logits, k)
    order = np.argsort(-logits, axis=1, kind="stable")
    assert np.array_equal(idx, order[:, :k])
    srt = np.take_along_axis(logits, order, axis=1)
    if k < E:
        assert np.array_equal(gap, srt[:, k - 1] - srt[:, k])
    else:
        assert np.all(np.isinf(gap))
    # weights: the full softmax renormalised over the selected set (scipy)
    full = scipy.special.softmax(logits, axis=1)
    sel = np.take_along_axis(full, idx.astype(np.int64), axis=1)
    assert np.allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-12, atol=0)


def test_topk_degenerate_weights():
    _, w, _ = oracle.topk(np.zeros((1, 16)), 16)
    assert np.allclose(w, 1.0 / 16, rtol=1e-15)
    _, w, _ = oracle.topk(np.random.default_rng(0).standard_normal((8, 16)), 1)
    assert np.all(w == 1.0)


def test_logits_closed_form_unit_router():
    # Wr row e = unit vector at column p[e]: logit_e = x[p[e]] + b[e] exactly.
    H, E = 64, 16
    rng = np.random.default_rng(2)
    p = rng.permutation(H)[:E]
    Wr = np.zeros((E, H), dtype=np.float32)
    Wr[np.arange(E), p] = 1.0
    b = rng.standard_normal(E).astype(np.float32)
    x = make_x(7, H, seed=2)
    _, _, _, logits = oracle.route(x, Wr, b, 3)
    xv = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(logits, xv[:, p] + b.astype(np.float64)[None, :])
    _, _, _, l0 = oracle.route(x, Wr, None, 3)
    assert np.array_equal(l0, xv[:, p])


def test_routing_invariants_full_size():
    cfg = MoeConfig("t", 2048, 512, 512, 10, 64, "zipf")
    Wr, b = make_router(cfg, seed=0)
    x = make_x(64, 2048, seed=0)
    idx, w, gap, logits = oracle.route(x, Wr, b, 10)
    for t in range(64):
        assert len(set(idx[t].tolist())) == 10
    assert idx.min() >= 0 and idx.max() < 512
    assert np.all(w > 0)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.diff(w, axis=1) <= 0)
    assert np.all(gap >= 0)


# ----------------------------------------------------------------------------
# the expert FFN and the layer


def _encode_matrix(d_rows_blocks, codes_rows_cols):
    """Canonical bytes for a matrix given fp16 scale per (row, block) and codes."""
    d = np.asarray(d_rows_blocks, dtype=np.float16)
    codes = np.asarray(codes_rows_cols, dtype=np.uint8)
    rows, cols = codes.shape
    out = []
    for r in range(rows):
        for bl in range(cols // 32):
            out.append(_block(int(d[r, bl:bl + 1].view(np.uint16)[0]), codes[r, bl * 32:(bl + 1) * 32]))
    return np.concatenate(out)


def _hand_expert(H=64, I=32):
    # gate row i: codes 2 (w = d), d = (i+1)/64 in both blocks -> g_i = i + 1 for x = 1
    gd = np.repeat(((np.arange(I) + 1) / 64.0)[:, None], H // 32, axis=1)
    gate = _encode_matrix(gd, np.full((I, H), 2))
    # up: block 0 codes 2 with d = 1/64, block 1 codes 0 (w = -d) with d = 1/128 -> u = 0.25
    ud = np.tile(np.array([1 / 64.0, 1 / 128.0]), (I, 1))
    uc = np.concatenate([np.full((I, 32), 2), np.full((I, 32), 0)], axis=1)
    up = _encode_matrix(ud, uc)
    # down row r: codes 3 (w = 2d), d = 2^-(r % 4) -> y_r = 2^(1 - r%4) * sum_i h_i
    dd = (2.0 ** -(np.arange(H) % 4))[:, None]
    down = _encode_matrix(dd, np.full((H, I), 3))
    return np.concatenate([gate, up, down])


def test_expert_hand_closed_form():
    H, I = 64, 32
    ex = _hand_expert(H, I)
    y = oracle.expert_forward(H, I, ex, np.ones(H))
    silu = lambda z: z / (1.0 + math.exp(-z))  # noqa: E731
    hsum = sum(silu(i + 1.0) * 0.25 for i in range(I))
    want = np.array([2.0 ** (1 - (r % 4)) * hsum for r in range(H)])
    assert np.allclose(y, want, rtol=1e-14, atol=0)
    # swapping the roles of gate and up would give silu(0.25) * (i+1): must differ
    wrong = sum(silu(0.25) * (i + 1.0) for i in range(I))
    assert abs(wrong - hsum) > 1.0


def test_layer_hand_closed_form():
    # Two experts plus shared, all equal to the hand expert; E=2, k=1, zero router.
    H, I = 64, 32
    ex = _hand_expert(H, I)
    experts = np.stack([ex, ex])
    Wr = np.zeros((2, H), dtype=np.float32)
    x = np.full((1, H), 0x3F80, dtype=np.uint16)  # bf16 1.0
    y, idx, w, gap = oracle.layer(x, Wr, None, experts, ex, top_k=1, inter=I)
    e_out = oracle.expert_forward(H, I, ex, np.ones(H))
    assert idx[0, 0] == 0 and w[0, 0] == 1.0 and gap[0] == 0.0  # tie -> lower index
    assert np.allclose(y[0], 2.0 * e_out, rtol=1e-15)


def _small_layer(H=64, I=32, E=8, k=3, T=5, seed=11):
    cfg = MoeConfig("t", H, I, E, k, T, "zipf")
    Wr, b = make_router(cfg, seed=seed)
    experts = np.stack([make_expert(H, I, seed, 0, e) for e in range(E)])
    shared = make_expert(H, I, seed, 0, E)
    x = make_x(T, H, seed=seed)
    return cfg, x, Wr, b, experts, shared


def test_layer_special_cases():
    cfg, x, Wr, b, experts, shared = _small_layer()
    H, I, E, k = cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k
    eb = experts.shape[1]
    y, idx, w, _ = oracle.layer(x, Wr, b, experts, shared, k, I)

    # all routed codes = 1 -> routed experts contribute exactly zero
    ez = experts.copy().reshape(E, eb // 10, 10)
    ez[:, :, 2:] = 0x55
    y_sh, _, _, _ = oracle.layer(x, Wr, b, ez.reshape(E, eb), shared, k, I)
    xs = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(cfg.tokens):
        assert np.array_equal(y_sh[t], oracle.expert_forward(H, I, shared, xs[t]))

    # all scales zero -> zero output
    e0 = experts.copy().reshape(E, eb // 10, 10)
    e0[:, :, 0:2] = 0
    s0 = shared.copy().reshape(eb // 10, 10)
    s0[:, 0:2] = 0
    y0, _, _, _ = oracle.layer(x, Wr, b, e0.reshape(E, eb), s0.reshape(-1), k, I)
    assert np.all(y0 == 0)

    # x = 0 -> zero output (no biases in the FFN)
    yz, _, _, _ = oracle.layer(np.zeros_like(x), Wr, b, experts, shared, k, I)
    assert np.all(yz == 0)

    # doubling every down-projection scale (exact in fp16) doubles y exactly
    down_off = 2 * I * H // 32
    e2 = experts.copy().reshape(E, eb // 10, 10)
    s2 = shared.copy().reshape(eb // 10, 10)
    for arr in (e2[:, down_off:], s2[None, down_off:]):
        d = np.ascontiguousarray(arr[..., 0:2]).view(np.float16)
        arr[..., 0:2] = (d.astype(np.float32) * 2).astype(np.float16).view(np.uint8)
    y2, _, _, _ = oracle.layer(x, Wr, b, e2.reshape(E, eb), s2.reshape(-1), k, I)
    assert np.array_equal(y2, 2.0 * y)

    # permuting experts together with router rows and bias leaves y unchanged
    perm = np.random.default_rng(4).permutation(E)
    yp, idxp, wp, _ = oracle.layer(x, Wr[perm], b[perm], experts[perm], shared, k, I)
    assert np.array_equal(yp, y)
    assert np.array_equal(perm[idxp], idx)
    assert np.array_equal(wp, w)


def test_layer_dense_equivalent():
    # Fully dequantised dense matrices (independent numpy decode), a dense
    # [T, E] gate matrix from scipy's softmax and numpy's stable argsort.
    cfg, x, Wr, b, experts, shared = _small_layer(H=128, I=64, E=16, k=4, T=9, seed=21)
    H, I, E, k = cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k
    y, idx, w, _ = oracle.layer(x, Wr, b, experts, shared, k, I)
    xs = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    logits = xs @ Wr.astype(np.float64).T + b.astype(np.float64)
    top = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    G = np.zeros((cfg.tokens, E))
    full = scipy.special.softmax(logits, axis=1)
    for t in range(cfg.tokens):
        G[t, top[t]] = full[t, top[t]] / full[t, top[t]].sum()
    gb = I * H // 32 * 10

    def ffn(ex):
        Wg = np_dequant(ex[:gb], I, H)
        Wu = np_dequant(ex[gb:2 * gb], I, H)
        Wd = np_dequant(ex[2 * gb:], H, I)
        g = xs @ Wg.T
        return (g / (1 + np.exp(-g)) * (xs @ Wu.T)) @ Wd.T

    want = ffn(shared) + sum(G[:, e:e + 1] * ffn(experts[e]) for e in range(E))
    assert np.array_equal(idx, top)
    assert np.max(np.abs(y - want)) <= 1e-12 * np.max(np.abs(want))


def test_layer_single_expert_is_textbook_swiglu():
    # E = 1, k = 1: y = shared(x) + expert(x), each a plain SwiGLU FFN (torch, fp64).
    cfg, x, Wr, b, experts, shared = _small_layer(H=96, I=64, E=1, k=1, T=4, seed=8)
    H, I = cfg.hidden, cfg.inter
    y, idx, w, _ = oracle.layer(x, Wr, b, experts, shared, 1, I)
    assert np.all(idx == 0) and np.all(w == 1.0)
    xs = torch.from_numpy((x.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    gb = I * H // 32 * 10

    def ffn(ex):
        Wg, Wu, Wd = (torch.from_numpy(np_dequant(ex[:gb], I, H)), torch.from_numpy(np_dequant(ex[gb:2 * gb], I, H)),
                      torch.from_numpy(np_dequant(ex[2 * gb:], H, I)))
        return torch.nn.functional.linear(torch.nn.functional.silu(xs @ Wg.T) * (xs @ Wu.T), Wd)

    want = (ffn(shared) + ffn(experts[0])).numpy()
    assert np.max(np.abs(y - want)) <= 1e-12 * np.max(np.abs(want))


def test_rmsnorm_pins():
    c = 3.0
    out = oracle.rmsnorm(np.full(2048, c), 1e-6)
    assert np.allclose(out, c / math.sqrt(c * c + 1e-6), rtol=1e-15)
    v = np.random.default_rng(0).standard_normal((4, 2048))
    want = torch.nn.functional.rms_norm(torch.from_numpy(v), (2048,), eps=1e-6).numpy()
    assert np.allclose(oracle.rmsnorm(v, 1e-6), want, rtol=1e-13, atol=0)


def test_bf16_input_encoding_is_rne():
    # the generator's float32 -> bf16 rounding agrees with torch's
    v = np.random.default_rng(3).standard_normal(10000).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(f32_to_bf16_bits(v), want)
