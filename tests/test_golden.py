"""The oracle and the workload shapes against the facts the pages state (tests/golden/, each file citing
its page and section)."""
import os

import numpy as np

import oracle
from gen import CONFIGS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    rows, kv = [], {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            a, b = line.split()
            try:
                rows.append((int(a), float(b)))
            except ValueError:
                kv[a] = float(b)
    return rows, kv


def _block(d_bits, q):
    blk = np.zeros(10, dtype=np.uint8)
    blk[0], blk[1] = d_bits & 0xFF, d_bits >> 8
    blk[2:] = (q & 3) * 0x55  # the same code in all four 2-bit fields of every byte
    return blk


def test_codebook_table():
    table, _ = _read("q2_affine_codebook.txt")
    assert [q for q, _ in table] == [0, 1, 2, 3]
    for d_bits in (0x3C00, 0x2E66, 0xBC00, 0x0400, 0x7BFF):
        d = float(np.array([d_bits], dtype=np.uint16).view(np.float16)[0])
        for q, wd in table:
            w = oracle.dequant_block(_block(d_bits, q))
            assert np.all(w == wd * d), (hex(d_bits), q)


def test_codebook_round_trip_difference():
    # Dequantise random blocks, re-encode every weight through the codebook (q = w / d + 1) and compare the
    # bytes and the weights: the largest difference must be the one the pages report.
    _, kv = _read("q2_affine_codebook.txt")
    rng = np.random.default_rng(7)
    n = 2000
    d = np.abs(rng.standard_normal(n).astype(np.float32) * 0.02).astype(np.float16)
    d[d == 0] = np.float16(1e-3)
    blocks = np.concatenate([d.view(np.uint8).reshape(n, 2), rng.integers(0, 256, size=(n, 8), dtype=np.uint8)], 1)
    W = oracle.dequant_matrix(blocks.reshape(-1), 1, n * 32).reshape(n, 32)
    q = np.rint(W / d.astype(np.float64)[:, None]).astype(np.int64) + 1
    re = np.zeros((n, 8), dtype=np.uint8)
    for j in range(32):
        re[:, j >> 2] |= (q[:, j].astype(np.uint8) & 3) << (2 * (j & 3))
    assert np.array_equal(re, blocks[:, 2:])
    diff = np.max(np.abs(W - d.astype(np.float64)[:, None] * (q - 1)))
    assert diff == kv["round_trip_max_abs_diff"]


def test_workload_shapes_follow_the_model_table():
    _, kv = _read("model_shape.txt")
    for name in ("decode", "prefill", "stack", "prefill_32k"):
        cfg = CONFIGS[name]
        assert cfg.n_experts == kv["routed_experts_per_layer"] and cfg.top_k == kv["active_routed_per_token"]
    assert CONFIGS["stack"].layers == kv["moe_layers"]
    assert kv["shared_experts"] == 1  # every layer here has exactly one shared expert (the `shared` argument)
