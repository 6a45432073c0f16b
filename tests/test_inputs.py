"""The seeded generator: shapes, determinism, value ranges, routing skew."""
import numpy as np

import oracle
from gen import CONFIGS, make_expert, make_router, make_x, canonical_expert_bytes


def test_shapes_and_determinism():
    cfg = CONFIGS["tiny"]
    x1, x2 = make_x(cfg, seed=0), make_x(cfg, seed=0)
    assert x1.shape == (8, 256) and x1.dtype == np.uint16 and np.array_equal(x1, x2)
    assert not np.array_equal(x1, make_x(cfg, seed=1))
    e = make_expert(cfg.hidden, cfg.inter, 0, 0, 3)
    assert e.size == canonical_expert_bytes(256, 128) == 3 * 256 * 128 // 32 * 10
    assert np.array_equal(e, make_expert(cfg.hidden, cfg.inter, 0, 0, 3))
    assert canonical_expert_bytes(2048, 512) == 983040


def test_code_and_scale_distribution():
    e = make_expert(2048, 512, 0, 0, 0).reshape(-1, 10)
    d = np.ascontiguousarray(e[:, :2]).view(np.float16)[:, 0].astype(np.float64)
    assert np.all(d >= 0)
    assert abs(d.mean() - 0.02 * np.sqrt(2 / np.pi)) < 2e-4     # E|N(0, s)| = s*sqrt(2/pi)
    codes = np.stack([(e[:, 2:] >> (2 * s)) & 3 for s in range(4)]).ravel()
    counts = np.bincount(codes, minlength=4) / codes.size
    assert np.all(np.abs(counts - 0.25) < 2e-3)


def test_zipf_skew_at_prefill_chunk():
    # T=1024, top-10 of 512: the hottest expert near 100 slots, every expert hit.
    cfg = CONFIGS["prefill"]
    Wr, b = make_router(cfg, seed=0)
    idx, w, gap, _ = oracle.route(make_x(cfg, seed=0), Wr, b, cfg.top_k)
    c = np.bincount(idx.ravel(), minlength=cfg.n_experts)
    assert c.sum() == 10240
    assert 80 <= c.max() <= 130
    assert c.min() >= 1
    # uniform routing at decode: bias zero
    Wr1, b1 = make_router(CONFIGS["decode"], seed=0)
    assert np.all(b1 == 0)
