"""Pins of the oracle's DSA comparison path and rotary embedding ("Token 的一生：
DSV4 架构与 DSpark" §1 从 DSA 到 DSV4: the DSA indexer selects top-k raw tokens;
§3.1 / §4: index Q and K go rope -> Hadamard -> quant in DSV4, DSA has no
Hadamard step), against facts outside the oracle's own arithmetic: hand-worked
rotations, the rotation being its own inverse, norm and relative-position
invariance, and dense causal attention when every key is selected."""
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
from oracle import oracle as orc  # noqa: E402


def test_rope_quarter_turn_by_hand():
    # freqs (cos, sin) = (0, 1) turns (a, b) into (-b, a); pairs past rope_dim untouched
    f = np.zeros((3, 2, 2))
    f[2, 0] = (0.0, 1.0)
    f[2, 1] = (1.0, 0.0)
    x = np.array([[1.0, 2.0, 3.0, 4.0, 5.0, 6.0]])
    np.testing.assert_array_equal(orc.rope(x, f, 4, [2]), [[-2.0, 1.0, 3.0, 4.0, 5.0, 6.0]])
    np.testing.assert_array_equal(orc.rope(x, f[:, :1], 2, [2]),
                                  [[-2.0, 1.0, 3.0, 4.0, 5.0, 6.0]])


def test_rope_half_turn_and_identity():
    f = np.zeros((2, 1, 2))
    f[0, 0] = (1.0, 0.0)
    f[1, 0] = (-1.0, 0.0)
    x = np.array([[0.5, -1.5, 7.0]])
    np.testing.assert_array_equal(orc.rope(x, f, 2, 0), x)
    np.testing.assert_array_equal(orc.rope(x, f, 2, 1), [[-0.5, 1.5, 7.0]])


def _table(max_pos, rd, base=10000.0):
    i = np.arange(rd // 2)
    a = np.arange(max_pos)[:, None] * base ** (-2.0 * i / rd)[None]
    return np.stack([np.cos(a), np.sin(a)], -1)


def test_rope_keeps_pair_norms_and_depends_on_relative_position():
    rng = np.random.default_rng(1)
    f = _table(64, 16)
    q, k = rng.standard_normal(24), rng.standard_normal(24)
    qr = orc.rope(q[None], f, 16, [10])[0]
    np.testing.assert_allclose(np.hypot(qr[0:16:2], qr[1:16:2]), np.hypot(q[0:16:2], q[1:16:2]),
                               rtol=1e-14)
    dots = [orc.rope(q[None], f, 16, [s + 7])[0] @ orc.rope(k[None], f, 16, [s])[0]
            for s in (0, 5, 40)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-12)


def test_dsa_quantise_is_index_quantise_of_the_rotated_row():
    # H/sqrt(n) is symmetric and orthogonal, so rotating twice is the identity:
    # quantising x without rotation equals index_quantise of rotate(x)
    rng = np.random.default_rng(2)
    for fmt in ("fp8", "fp4", "bf16"):
        x = rng.standard_normal((20, 128))
        a = orc.dsa_index_quantise(x, fmt)
        b = orc.index_quantise(orc.hadamard_rotate(x), fmt)
        np.testing.assert_array_equal(a["codes"], b["codes"])
        np.testing.assert_allclose(a["deq"], b["deq"], rtol=0, atol=0)
    # and a row already on the FP8 grid comes back exactly
    # codes 0..126 (126 = 448, the largest finite E4M3) times 0.5: scale 224/448
    g = np.array([orc.e4m3_value(c) for c in range(0, 127)])[None] * 0.5
    g = np.concatenate([g, np.zeros((1, 1))], 1)
    np.testing.assert_array_equal(orc.dsa_index_quantise(g, "fp8")["deq"], g)


def test_dsa_step_selects_everything_when_short():
    # with L <= 512 every visible raw token is selected, so each query's output
    # is dense causal attention over tokens 0..p (float64 SDPA)
    from compressed_sparse_attention_12_b200 import synth
    w = synth.workload("dsa_128k", 1 / 512)       # L = 256 per request
    w.seq_lens[:] = 300
    w.q_lens[:] = 1
    d = synth.draw_dsa(w, "cpu")
    pt = synth.dsa_page_table(w)
    r = orc.dsa_step(w, d, pt, requests=[0, 3])
    for t in (0, 3):
        assert r[t]["n_vis"] == 300
        assert np.array_equal(r[t]["logical"][:300], np.arange(300))
        assert (r[t]["logical"][300:] == -1).all()
        # physical index through the 64-token page table
        assert np.array_equal(r[t]["phys"][:300], pt[t, np.arange(300) // 64] * 64 +
                              np.arange(300) % 64)
        rows = orc.kv_decode_rows(orc.kv_encode_rows(d["kv"][300 * t:300 * t + 300].double()
                                                     .numpy(), True), True)
        k = torch.tensor(rows)
        want = torch.nn.functional.scaled_dot_product_attention(
            d["q"][t].double()[None, None], k[None, None], k[None, None, :, :512],
            scale=1 / 24)[0, 0].numpy()
        np.testing.assert_allclose(r[t]["out"], want, rtol=1e-10, atol=1e-10)


def test_rope_golden():
    import json
    path = os.path.join(os.path.dirname(__file__), "golden", "rope_example.json")
    with open(path) as f:
        gold = json.load(f)
    f = np.array(gold["freqs"], dtype=np.float64)
    x = np.array([gold["x"]], dtype=np.float64)
    for case in gold["cases"]:
        y = orc.rope(x, f, gold["rope_dim"], [case["pos"]])
        np.testing.assert_allclose(y[0], case["y"], rtol=0, atol=1e-15)
