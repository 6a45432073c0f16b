"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, MoeConfig, make_x
from parity import GAP_TIE, W_TOL, build_layer, check_layer, check_routing, gpu_forward, to_dev_bf16


def bf16_to_f32(bits):
    return (np.asarray(bits).view(np.uint16).astype(np.uint32) << 16).view(np.float32)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__

    __graft_entry__.build()
    assert torch.cuda.is_available()


@pytest.fixture(scope="module")
def tiny():
    return build_layer(CONFIGS["tiny"])


@pytest.fixture(scope="module")
def full():
    return build_layer(CONFIGS["prefill"])  # full-size layer with the Zipf router bias


@pytest.mark.parametrize("T", [1, 2, 3, 7, 8, 9, 33, 100, 257])
def test_tiny_layer_all_tokens(tiny, T):
    L, w = tiny
    x = make_x(T, 256, seed=100 + T)
    y, idx, wts = gpu_forward(L, x)
    err, l2, flagged = check_layer(CONFIGS["tiny"], w, x, y, idx, wts)
    assert l2 < 5e-3


def test_tiny_layer_exact_workload(tiny):
    L, w = tiny
    x = make_x(CONFIGS["tiny"], seed=0)
    y, idx, wts = gpu_forward(L, x)
    check_layer(CONFIGS["tiny"], w, x, y, idx, wts)


@pytest.mark.parametrize("dims", [(384, 256, 8, 3), (256, 128, 1, 1), (256, 128, 16, 16), (128, 384, 32, 5),
                                  (1024, 128, 64, 8), (512, 512, 16, 2)])
def test_odd_shapes(dims):
    H, I, E, k = dims
    cfg = MoeConfig("t", H, I, E, k, 13, "zipf")
    L, w = build_layer(cfg, seed=3)
    for T in (1, 13):
        x = make_x(T, H, seed=T)
        y, idx, wts = gpu_forward(L, x)
        check_layer(cfg, w, x, y, idx, wts)


def test_many_experts_beyond_the_fused_kernel():
    """5000 routed experts (above the fused decode kernel's 1024): T = 3 takes the routing kernels plus the
    register-dequant expert kernels, T = 13 and 300 the tcgen05 path; E near the 65535 limit only grows the
    same per-expert work lists."""
    cfg = MoeConfig("many experts", 128, 128, 5000, 4, 13, "zipf")
    L, w = build_layer(cfg, seed=5)
    for T in (3, 13, 300):
        x = make_x(T, 128, seed=50 + T)
        y, idx, wts = gpu_forward(L, x)
        err, l2, flagged = check_layer(cfg, w, x, y, idx, wts)
        print(f"E=5000 T={T}: max-rel {err:.3e} relL2 {l2:.3e} flagged {len(flagged)}")


def test_decode_window_full_size(full):
    L, w = full
    cfg = CONFIGS["decode"]
    for T in (1, 2, 3):
        x = make_x(T, cfg.hidden, seed=7)
        y, idx, wts = gpu_forward(L, x)
        err, l2, flagged = check_layer(cfg, w, x, y, idx, wts)
        print(f"T={T}: max-rel {err:.3e} relL2 {l2:.3e} flagged {len(flagged)}")


def test_decode_layer_uniform_router():
    cfg = CONFIGS["decode"]
    L, w = build_layer(cfg)
    x = make_x(cfg, seed=0)
    y, idx, wts = gpu_forward(L, x)
    err, l2, flagged = check_layer(cfg, w, x, y, idx, wts)
    print(f"decode layer: max-rel {err:.3e} relL2 {l2:.3e}")


def test_prefill_chunk_1024(full):
    cfg = CONFIGS["prefill"]
    L, w = full
    x = make_x(cfg, seed=0)
    y, idx, wts = gpu_forward(L, x)
    # routing: every token against the oracle
    idx_o, w_o, gap, _ = oracle.route(x, w["router_w"], w["router_b"], cfg.top_k)
    flagged = check_routing(idx, wts, idx_o, w_o, gap)
    # outputs: every token
    err, l2, _ = check_layer(cfg, w, x, y, idx, wts)
    print(f"prefill chunk 1024: max-rel {err:.3e} relL2 {l2:.3e} flagged {len(flagged)}")


@pytest.mark.parametrize("T", [600, 1500])
def test_prefill_many_tokens_per_expert(T):
    """Experts averaging 64 or more tokens take the one-tile, 128-token work items (ragged last items)."""
    cfg = MoeConfig("many", 256, 128, 16, 2, T, "zipf")
    L, w = build_layer(cfg, seed=7)
    x = make_x(T, 256, seed=T)
    y, idx, wts = gpu_forward(L, x)
    err, l2, flagged = check_layer(cfg, w, x, y, idx, wts)
    print(f"many-token items T={T}: max-rel {err:.3e} relL2 {l2:.3e} flagged {len(flagged)}")
    assert l2 < 5e-3


def test_prefill_ragged_and_cold_tail():
    cfg = MoeConfig("cold", 2048, 512, 512, 10, 133, "zipf_cold")
    L, w = build_layer(cfg, seed=1)
    x = make_x(cfg, seed=1)
    y, idx, wts = gpu_forward(L, x)
    check_layer(cfg, w, x, y, idx, wts)


@pytest.mark.parametrize("cold", [0, 8])
def test_verify_windows_and_cold_tail_per_expert_kernels(cold):
    """Wider verify windows (T = 16, 32, 64 tokens: --spec 4/6/8 windows, Strata tuning page sections 5 and 8) and
    the cold-tail router (many experts with 1-2 tokens), every token against the oracle, with every expert on the
    tcgen05 kernels (cold = 0, the default) and with experts of at most 8 tokens on the register-dequant kernels
    (cold = 8, moe_set_cold_expert_tokens)."""
    from bit_block_quantized_moe_b200 import moe_set_cold_expert_tokens

    moe_set_cold_expert_tokens(cold)
    try:
        for bias, Ts in (("zipf", (16, 32, 64)), ("zipf_cold", (133, 1024))):
            cfg = MoeConfig("windows", 2048, 512, 512, 10, 64, bias)
            L, w = build_layer(cfg, seed=2)
            for T in Ts:
                x = make_x(T, 2048, seed=60 + T)
                y, idx, wts = gpu_forward(L, x)
                err, l2, flagged = check_layer(cfg, w, x, y, idx, wts)
                counts = np.bincount(idx.ravel(), minlength=512)
                print(f"cold={cold} {bias} T={T}: max-rel {err:.3e} relL2 {l2:.3e} flagged {len(flagged)}; experts "
                      f"with <= 8 tokens: {int(((counts > 0) & (counts <= 8)).sum())}")
            del L
    finally:
        moe_set_cold_expert_tokens(0)


def test_route_entry_point(full):
    L, w = full
    cfg = CONFIGS["prefill"]
    for T in (3, 1024):
        x = make_x(T, cfg.hidden, seed=11)
        idx, wts = L.route(to_dev_bf16(x))
        torch.cuda.synchronize()
        idx_o, w_o, gap, _ = oracle.route(x, w["router_w"], w["router_b"], cfg.top_k)
        check_routing(idx.cpu().numpy(), wts.cpu().numpy(), idx_o, w_o, gap)


def test_deterministic_and_zero_tokens(tiny):
    L, w = tiny
    x = make_x(100, 256, seed=5)
    y1, i1, w1 = gpu_forward(L, x)
    y2, i2, w2 = gpu_forward(L, x)
    assert np.array_equal(y1, y2) and np.array_equal(i1, i2) and np.array_equal(w1, w2)
    out = torch.full((1, 256), 7, dtype=torch.int16, device="cuda")
    L.forward(torch.empty((0, 256), dtype=torch.int16, device="cuda"), out=out[:0])
    torch.cuda.synchronize()
    assert torch.all(out == 7)


def test_rmsnorm_residual():
    from bit_block_quantized_moe_b200 import moe_rmsnorm_residual

    T, H = 37, 2048
    rng = np.random.default_rng(0)
    resid = rng.standard_normal((T, H)).astype(np.float32)
    y = make_x(T, H, seed=9)
    r_d = torch.from_numpy(resid.copy()).cuda()
    y_d = to_dev_bf16(y)
    xn = torch.empty((T, H), dtype=torch.int16, device="cuda")
    moe_rmsnorm_residual(r_d, y_d, xn, T, H, 1e-6)
    torch.cuda.synchronize()
    r_ref = resid.astype(np.float64) + (y.astype(np.uint32) << 16).view(np.float32)
    assert np.max(np.abs(r_d.cpu().numpy() - r_ref)) < 1e-5
    want = oracle.rmsnorm(r_ref, 1e-6)
    got = (xn.cpu().numpy().view(np.uint16).astype(np.uint32) << 16).view(np.float32)
    assert np.max(np.abs(got - want) / np.maximum(np.abs(want), 1e-3)) < 2 ** -8


def test_experts_forward_given_routing(tiny):
    L, w = tiny
    cfg = CONFIGS["tiny"]
    T = 21
    x = make_x(T, 256, seed=3)
    rng = np.random.default_rng(0)
    forced = np.stack([rng.choice(16, 2, replace=False) for _ in range(T)]).astype(np.int32)
    y_o, _, w_o, _ = oracle.layer(x, w["router_w"], w["router_b"], w["experts"], w["shared"], 2, 128,
                                  forced_idx=forced)
    out = L.experts_forward(to_dev_bf16(x), torch.from_numpy(forced).cuda(),
                            torch.from_numpy(w_o.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    L.check_status()
    y = (out.cpu().numpy().view(np.uint16).astype(np.uint32) << 16).view(np.float32)
    assert np.max(np.abs(y - y_o)) / np.max(np.abs(y_o)) <= 1e-2


def test_experts_forward_bad_index_sets_status(tiny):
    from bit_block_quantized_moe_b200 import MoeError

    L, w = tiny
    T = 4
    x = make_x(T, 256, seed=4)
    idx = torch.tensor([[0, 1], [2, 99], [3, 4], [-5, 6]], dtype=torch.int32, device="cuda")
    wt = torch.full((T, 2), 0.5, dtype=torch.float32, device="cuda")
    L.experts_forward(to_dev_bf16(x), idx, wt)
    with pytest.raises(MoeError) as ei:
        L.check_status()
    assert ei.value.code == 6  # MOE_ERR_DEVICE
    L.check_status()  # cleared


@pytest.mark.parametrize("T", [2, 3, 4])
def test_fused_decode_repeated_experts(full, T):
    """Identical tokens choose the same experts, so every expert is chosen by all T tokens: T <= 3 streams it
    once per (token, slot) entry, T = 4 once per touched expert.  Against the oracle, and the output rows are
    equal bit for bit (each token's contributions are summed in the same order)."""
    L, w = full
    x1 = make_x(1, 2048, seed=55)
    x = np.repeat(x1, T, axis=0)
    y, idx, wts = gpu_forward(L, x)
    assert all(np.array_equal(idx[t], idx[0]) and np.array_equal(wts[t], wts[0]) for t in range(T))
    assert all(np.array_equal(y[t], y[0]) for t in range(T))
    err, l2, flagged = check_layer(CONFIGS["prefill"], w, x, y, idx, wts)
    print(f"repeated experts T={T}: max-rel {err:.3e} relL2 {l2:.3e}")


def test_fused_decode_barrier_counter(full):
    """The fused kernel's two grid barriers each add one arrival per CTA to the workspace's monotonic counter
    (offset 64), so every launch moves it by exactly twice the grid size (one CTA per SM) whatever T, and the
    barrier targets a launch derives from the value it reads at start stay right across a run of mixed window
    sizes on one workspace."""
    L, w = full
    L.reserve(8)
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count

    def counter():
        torch.cuda.synchronize()
        return int(L.workspace[64:72].cpu().numpy().view(np.uint64)[0])

    c = counter()
    assert c % n_sm == 0
    for i, T in enumerate((3, 1, 8, 2, 5, 3)):
        x = make_x(T, 2048, seed=900 + i)
        y, idx, wts = gpu_forward(L, x)
        c2 = counter()
        assert c2 - c == 2 * n_sm, (T, c, c2)
        c = c2
        check_layer(CONFIGS["prefill"], w, x, y, idx, wts)


def test_layer_forward_host_memory(full):
    """moe_layer_forward_host: the token rows read from and the output written to page-locked host memory by
    the library's copy kernels in stream order, equal bit for bit to moe_layer_forward on device buffers
    (routing copies too); several steps back to back on one stream with no synchronisation between them (the
    copy-in of a step is launched while the previous step still runs) and each against the oracle."""
    from bit_block_quantized_moe_b200 import MoeError, moe_layer_forward_host

    L, w = full
    L.reserve(8)
    stream = torch.cuda.Stream()
    steps = [(3, 301), (1, 302), (8, 303), (3, 304), (2, 305)]
    xh = [torch.from_numpy(make_x(T, 2048, seed=sd).view(np.int16)).pin_memory() for T, sd in steps]
    oh = [torch.zeros((T, 2048), dtype=torch.int16).pin_memory() for T, _ in steps]
    ih = [torch.full((T, 10), -1, dtype=torch.int32, device="cuda") for T, _ in steps]
    wh = [torch.zeros((T, 10), dtype=torch.float32, device="cuda") for T, _ in steps]
    with torch.cuda.stream(stream):
        for i in range(len(steps)):
            L.forward_host(xh[i], oh[i], topk_idx=ih[i], topk_w=wh[i], stream=stream)
    stream.synchronize()
    L.check_status()
    for i, (T, _) in enumerate(steps):
        x = xh[i].numpy()
        y_ref, idx_ref, w_ref = gpu_forward(L, x)
        y = bf16_to_f32(oh[i].numpy()).astype(np.float64)
        assert np.array_equal(y, y_ref), T
        assert np.array_equal(ih[i].cpu().numpy(), idx_ref) and np.array_equal(wh[i].cpu().numpy(), w_ref)
        check_layer(CONFIGS["prefill"], w, x.view(np.uint16), y, idx_ref, w_ref)
    # pageable host memory, device memory and windows over 8 tokens are refused before any launch
    pageable = torch.from_numpy(make_x(3, 2048, seed=1).view(np.int16))
    for bad_x, bad_out, T in ((pageable, oh[0], 3), (xh[0], torch.zeros((3, 2048), dtype=torch.int16), 3),
                              (xh[0].cuda(), oh[0], 3)):
        with pytest.raises(MoeError) as e:
            moe_layer_forward_host(L.dims, bad_x, L.router_w, L.router_b, L.experts, L.shared, bad_out, T,
                                   L.workspace)
        assert e.value.code == 1  # MOE_ERR_ARG
    x9 = torch.from_numpy(make_x(9, 2048, seed=2).view(np.int16)).pin_memory()
    o9 = torch.zeros((9, 2048), dtype=torch.int16).pin_memory()
    L.reserve(9)
    with pytest.raises(MoeError) as e:
        moe_layer_forward_host(L.dims, x9, L.router_w, L.router_b, L.experts, L.shared, o9, 9, L.workspace)
    assert e.value.code == 1
    L.check_status()


@pytest.mark.parametrize("T", [4, 5, 8])
def test_fused_decode_window_sizes(full, T):
    L, w = full
    x = make_x(T, 2048, seed=40 + T)
    y, idx, wts = gpu_forward(L, x)
    err, l2, flagged = check_layer(CONFIGS["prefill"], w, x, y, idx, wts)
    print(f"fused T={T}: max-rel {err:.3e} relL2 {l2:.3e}")


def test_fused_decode_agrees_with_route_and_general_path(full):
    L, w = full
    T = 3
    x = make_x(T, 2048, seed=77)
    xd = to_dev_bf16(x)
    y1, idx1, w1 = gpu_forward(L, x)
    y2, idx2, w2 = gpu_forward(L, x)
    assert np.array_equal(y1, y2) and np.array_equal(idx1, idx2)  # deterministic
    ridx, rw = L.route(xd)
    torch.cuda.synchronize()
    assert np.array_equal(ridx.cpu().numpy(), idx1) and np.array_equal(rw.cpu().numpy(), w1)
    out = L.experts_forward(xd, ridx, rw)  # general dispatch path, same routing
    torch.cuda.synchronize()
    yg = (out.cpu().numpy().view(np.uint16).astype(np.uint32) << 16).view(np.float32)
    assert np.max(np.abs(yg - y1)) <= 4e-3 * np.max(np.abs(y1))


def test_routing_copies_one_at_a_time(full):
    """moe_layer_forward asked for only one of the two routing copies (the fused decode path writes them as a
    pair; the other goes to the workspace)."""
    L, w = full
    x = make_x(3, 2048, seed=91)
    xd = to_dev_bf16(x)
    ridx, rw = L.route(xd)
    idx = torch.full((3, 10), -1, dtype=torch.int32, device="cuda")
    y1 = L.forward(xd, topk_idx=idx)
    wts = torch.zeros((3, 10), dtype=torch.float32, device="cuda")
    y2 = L.forward(xd, topk_w=wts)
    torch.cuda.synchronize()
    L.check_status()
    assert torch.equal(idx, ridx) and torch.equal(wts, rw)
    assert torch.equal(y1, y2)


def _stack_against_oracle(L, fused, assert_trajectory=True):
    """A stack of L full-size layers at T = 1024, end to end: x_0 = x; layer l reads bf16(RMSNorm(r_l));
    r_{l+1} = r_l + y_l, the residual fp32 on the GPU and fp64 in the oracle.  The GPU runs all 1024 tokens
    through all L layers with no re-anchoring (fused: moe_layer_forward_residual; else moe_layer_forward +
    moe_rmsnorm_residual); the oracle stack carries 256 sampled tokens through the same layers from the same x.

    Every routing decision the GPU takes is checked against the oracle's routing of the GPU's own layer input
    (sets bit-exact except near-ties).  The two trajectories' layer inputs drift apart by the accumulated
    rounding of earlier layers, so a token whose margin is below that drift may take a different set on the two
    sides; there the oracle stack takes the GPU's set (counted and printed).  The final residuals must agree
    within max|dr| / max|r| <= 1e-2; the drift of the bf16 layer input is printed every 8 layers."""
    import math

    from bit_block_quantized_moe_b200 import moe_rmsnorm_residual
    from gen import make_layer

    cfg = CONFIGS["stack"]
    T, H, k = cfg.tokens, cfg.hidden, cfg.top_k
    rng = np.random.default_rng(3)
    sample = np.sort(rng.choice(T, 256, replace=False))
    x0 = make_x(cfg, seed=0)
    resid = torch.from_numpy(bf16_to_f32(x0)).cuda()
    xn = torch.empty((T, H), dtype=torch.int16, device="cuda")
    xn2 = torch.empty_like(xn)
    moe_rmsnorm_residual(resid, None, xn, T, H, 1e-6)
    idx_g = np.empty((L, sample.size, k), dtype=np.int32)
    w_g = np.empty((L, sample.size, k), dtype=np.float32)
    xn_g = np.empty((L, sample.size, H), dtype=np.uint16)
    y_g = np.empty((L, sample.size, H), dtype=np.float64)
    for layer in range(L):
        Lyr, _ = build_layer(cfg, layer=layer)
        idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        wts = torch.zeros((T, k), dtype=torch.float32, device="cuda")
        xn_g[layer] = xn.cpu().numpy().view(np.uint16)[sample]
        if fused:
            Lyr.forward_residual(xn, resid, xn2, 1e-6, topk_idx=idx, topk_w=wts)
            xn, xn2 = xn2, xn
        else:
            y = Lyr.forward(xn, topk_idx=idx, topk_w=wts)
            y_g[layer] = bf16_to_f32(y.cpu().numpy().view(np.uint16)[sample])
            moe_rmsnorm_residual(resid, y, xn, T, H, 1e-6)  # r += y; the next layer's input
        torch.cuda.synchronize()
        Lyr.check_status()
        idx_g[layer] = idx.cpu().numpy()[sample]
        w_g[layer] = wts.cpu().numpy()[sample]
        del Lyr
    torch.cuda.synchronize()
    r_gpu = resid.cpu().numpy()[sample].astype(np.float64)

    r = None
    followed, flagged = 0, 0
    bounds = sorted(set(list(range(0, L, 8)) + [max(L - 1, 0), L]))
    for c0, c1 in zip(bounds[:-1], bounds[1:]):
        lays = [make_layer(cfg, seed=0, layer=l) for l in range(c0, c1)]
        # the layer input of layer c0 on both sides
        u_o = bf16_to_f32(oracle.double_to_bf16(oracle.rmsnorm(bf16_to_f32(x0[sample]).astype(np.float64)
                                                               if r is None else r, 1e-6)))
        u_g = bf16_to_f32(xn_g[c0])
        print(f"stack layer {c0:2d} input: max|du|/max|u| = {np.max(np.abs(u_g - u_o)) / np.max(np.abs(u_o)):.3e}")
        for l, lay in zip(range(c0, c1), lays):  # every GPU routing decision, on the GPU's own layer input
            idx_o, w_o, gap, _ = oracle.route(xn_g[l], lay["router_w"], lay["router_b"], k)
            flagged += len(check_routing(idx_g[l], w_g[l], idx_o, w_o, gap))
            if not fused:  # each layer's bf16 output against the oracle layer on the GPU's own input
                err_l, _, _ = check_layer(cfg, lay, xn_g[l], y_g[l], idx_g[l], w_g[l])
                print(f"stack layer {l} output on its own input: max-rel {err_l:.3e}")
        r, _, _, nf, nm = oracle.stack(x0[sample], lays, k, cfg.inter, eps=1e-6, follow_idx=idx_g[c0:c1],
                                       tie_gap=math.inf, resid_in=r)
        followed += nf
        del lays
    err = np.max(np.abs(r_gpu - r)) / np.max(np.abs(r))
    rel_l2 = np.linalg.norm(r_gpu - r) / np.linalg.norm(r)
    print(f"stack of {L} layers ({'fused residual' if fused else 'layer + rmsnorm_residual'}), 256 tokens: final "
          f"residual max|dr|/max|r| = {err:.3e}, relL2 {rel_l2:.3e}; near-tie routing differences on the GPU's own "
          f"inputs: {flagged}; (layer, token) pairs where the two trajectories routed differently and the oracle "
          f"took the GPU's set: {followed} of {L * sample.size}")
    if assert_trajectory:
        assert err <= 1e-2


def test_stack_48_layers_against_oracle_stack():
    """The pages' model depth: 48 layers (Strata tuning page, section 2 model table), through the fused
    residual call the stack benchmark times."""
    _stack_against_oracle(48, fused=True)


def test_stack_6_layers_layer_plus_rmsnorm_against_oracle_stack():
    """The same stack composed of moe_layer_forward + moe_rmsnorm_residual, which rounds each layer output to bf16
    before the residual takes it.  Every layer output is checked against the oracle layer on the GPU's own input
    (max-rel <= 1e-2); the trajectory against the fp64 oracle stack is printed, not asserted: with the output
    rounded to bf16 it drifts past 1e-2 within a few layers (3.6e-2 after 6 measured on B200), which is why the
    stack's own entry point (moe_layer_forward_residual, checked over 48 layers above) adds the output unrounded."""
    _stack_against_oracle(6, fused=False, assert_trajectory=False)


@pytest.mark.parametrize("T", [3, 5, 100, 1024])
def test_layer_forward_residual(full, T):
    """resid += layer(x_norm) and the next RMSNorm in the layer's last kernel: against moe_layer_forward +
    moe_rmsnorm_residual (which rounds y to bf16 first) and against the oracle's layer output."""
    from bit_block_quantized_moe_b200 import moe_rmsnorm_residual

    L, w = full
    cfg = CONFIGS["prefill"]
    H = cfg.hidden
    rng = np.random.default_rng(T)
    r0 = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).cuda()
    xn = torch.empty((T, H), dtype=torch.int16, device="cuda")
    moe_rmsnorm_residual(r0.clone(), None, xn, T, H, 1e-6)
    ra, xa = r0.clone(), torch.empty_like(xn)
    idx = torch.full((T, cfg.top_k), -1, dtype=torch.int32, device="cuda")
    wts = torch.zeros((T, cfg.top_k), dtype=torch.float32, device="cuda")
    L.forward_residual(xn, ra, xa, 1e-6, topk_idx=idx, topk_w=wts)
    y = L.forward(xn)
    rb, xb = r0.clone(), torch.empty_like(xn)
    moe_rmsnorm_residual(rb, y, xb, T, H, 1e-6)
    torch.cuda.synchronize()
    L.check_status()
    ya = (ra - r0).cpu().numpy().astype(np.float64)
    ymax = float(np.max(np.abs(ya)))
    # the unfused pair differs only by y's bf16 rounding
    assert torch.max(torch.abs(ra - rb)).item() <= 2.0 ** -8 * ymax + 1e-6
    xn_np = xn.cpu().numpy().view(np.uint16)
    err, l2, flagged = check_layer(cfg, w, xn_np, ya, idx.cpu().numpy(), wts.cpu().numpy())
    want = oracle.rmsnorm(ra.cpu().numpy().astype(np.float64), 1e-6)
    got = bf16_to_f32(xa.cpu().numpy().view(np.uint16))
    assert np.max(np.abs(got - want) / np.maximum(np.abs(want), 1e-3)) < 2 ** -8
    print(f"fused residual T={T}: layer max-rel {err:.3e} relL2 {l2:.3e} flagged {len(flagged)}")


def test_prefill_chunk_32768(full):
    """A T = 32768 prefill chunk through a full-size Zipf layer: routing of
    every token against the oracle, outputs on 256 sampled tokens (plus the flagged
    ones and both ends).  The decode sweep T in {1, 2, 3} on the same weights is
    test_decode_window_full_size."""
    cfg = CONFIGS["prefill_32k"]
    L, w = full
    x = make_x(cfg, seed=4)
    y, idx, wts = gpu_forward(L, x)
    idx_o, w_o, gap, _ = oracle.route(x, w["router_w"], w["router_b"], cfg.top_k)
    flagged = check_routing(idx, wts, idx_o, w_o, gap)
    rng = np.random.default_rng(4)
    sample = np.union1d(rng.choice(cfg.tokens, 256, replace=False), np.array(flagged, dtype=np.int64))
    sample = np.union1d(sample, [0, cfg.tokens - 1])
    err, l2, _ = check_layer(cfg, w, x, y, idx, wts, tokens=sample)
    print(f"prefill chunk 32768: max-rel {err:.3e} relL2 {l2:.3e} flagged {len(flagged)}")
