"""Pins of the HCA oracle ("DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", section
"Heavily Compressed Attention（HCA）": about 128x compression, dense attention
over the compressed blocks) against facts that do not depend on the oracle's
own arithmetic: the C4 compressor (pinned separately) as the ratio-4 case,
one-hot and flat gates, the zero-gate closed form, and torch's SDPA in float64
for the dense attention."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc


def test_pool_ratio4_is_the_c4_compressor():
    rng = np.random.default_rng(1)
    x, g = rng.standard_normal((2 * 4 * 9 + 3, 16)), rng.standard_normal((2 * 4 * 9 + 3, 16))
    b = rng.standard_normal((4, 16))
    np.testing.assert_allclose(orc.pool_compress(x, g, b, 4), orc.c4_compress(x, g, b),
                               rtol=0, atol=1e-13)


def test_hca_one_hot_gate_copies_the_chosen_row():
    rng = np.random.default_rng(2)
    T, D = 3 * 128 + 50, 24
    x = rng.standard_normal((T, D))
    g = np.full((T, D), -80.0)
    pick = rng.integers(0, 128, size=(T // 128, D))
    for j in range(T // 128):
        for c in range(D):
            g[128 * j + pick[j, c], c] = 80.0
    y = orc.hca_compress(x, g, np.zeros((128, D)))
    assert y.shape == (3, D)
    want = np.array([[x[128 * j + pick[j, c], c] for c in range(D)] for j in range(3)])
    np.testing.assert_allclose(y, want, rtol=0, atol=1e-12)


def test_hca_flat_gate_is_the_block_mean():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((256, 8))
    y = orc.hca_compress(x, np.full((256, 8), 0.7), np.zeros((128, 8)))
    np.testing.assert_allclose(y, x.reshape(2, 128, 8).mean(axis=1), rtol=0, atol=1e-13)


def test_hca_zero_gate_weights_are_the_bias_softmax():
    # with g = 0 the weights of position i are exp(b_i) / sum_k exp(b_k), the
    # same for every block
    rng = np.random.default_rng(4)
    x = rng.standard_normal((384, 4))
    b = rng.standard_normal((128, 4)) * 2.0
    wgt = np.exp(b) / np.exp(b).sum(axis=0, keepdims=True)
    want = (x.reshape(3, 128, 4) * wgt[None]).sum(axis=1)
    np.testing.assert_allclose(orc.hca_compress(x, np.zeros_like(x), b), want, rtol=1e-12,
                               atol=1e-13)


def test_hca_lengths():
    assert [orc.hca_len(L) for L in (0, 127, 128, 255, 256, 1048576)] == [0, 0, 1, 1, 2, 8192]
    assert [orc.hca_visible(p) for p in (0, 126, 127, 128, 255)] == [0, 0, 1, 1, 2]


def test_hca_attention_single_row_returns_its_value():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4, 576))
    row = rng.standard_normal((1, 576))
    out, lse = orc.hca_attention(q, row, np.zeros((0, 576)), 0.1)
    np.testing.assert_allclose(out, np.repeat(row[:, :512], 4, axis=0), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, 0.1 * q @ row[0], rtol=1e-14)


@pytest.mark.parametrize("n_hca,n_win", [(5, 0), (64, 128), (1, 3)])
def test_hca_attention_matches_sdpa(n_hca, n_win):
    rng = np.random.default_rng(n_hca + n_win)
    H = 8
    q = rng.standard_normal((H, 576))
    hrows = rng.standard_normal((n_hca, 576))
    wrows = rng.standard_normal((n_win, 576))
    out, lse = orc.hca_attention(q, hrows, wrows, 1 / 24)
    k = torch.tensor(np.concatenate([hrows, wrows]), dtype=torch.float64)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q, dtype=torch.float64)[None, None], k[None, None], k[None, None, :, :512],
        scale=1 / 24)[0, 0].numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    s = (q @ k.numpy().T) / 24
    np.testing.assert_allclose(lse, np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) +
                               s.max(1), rtol=1e-12)


def test_hca_step_flat_gate_block_is_the_mean_and_rows_follow_visibility():
    # a whole oracle HCA step on a small workload with the compressor's gate and
    # bias set flat: the freshly pooled row is the block mean, so every query's
    # output equals dense attention over [drawn rows, block mean] cut at
    # hca_visible(p), plus its window
    import sys, os
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
    from compressed_sparse_attention_12_b200 import synth
    w = synth.workload("hca_prefill", 1 / 16)
    d = synth.draw_hca(w, "cpu")
    d["gate"] = torch.zeros_like(d["gate"])
    d["bias"] = torch.zeros_like(d["bias"])
    pt = synth.page_table(w)
    ref = orc.hca_step(w, d, pt)
    L, Q = int(w.seq_lens[0]), int(w.q_lens[0])
    direct = d["hca_kv"].double().numpy()
    new = d["raw_kv"].double().numpy()
    assert new.shape[0] % 128 == 0 and new.shape[0] > 0
    rows = np.concatenate([direct, new.reshape(-1, 128, 576).mean(axis=1)])
    assert rows.shape[0] == L // 128
    deq = orc.kv_decode_rows(orc.kv_encode_rows(rows, True), True)
    raw = dict(zip(d["raw_pos"].tolist(),
                   orc.kv_decode_rows(orc.kv_encode_rows(d["kv_raw"].double().numpy(), True), True)))
    q = d["q"].double().numpy()
    for j in (0, Q // 2, Q - 1):
        p = L - Q + j
        nv = (p + 1) // 128
        assert ref[j]["n_hca"] == nv
        win = np.array([raw[r] for r in range(max(0, p - w.window + 1), p + 1)])
        k = torch.tensor(np.concatenate([deq[:nv], win]))
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q[j])[None, None], k[None, None], k[None, None, :, :512],
            scale=1 / 24)[0, 0].numpy()
        np.testing.assert_allclose(ref[j]["out"], want, rtol=1e-10, atol=1e-10)


def test_hca_pool_golden():
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "hca_pool_example.json")
    with open(path) as f:
        gold = json.load(f)
    for case in gold["cases"]:
        x = np.array(case["x"], dtype=np.float64)[:, None]
        g = np.array(case["gate"], dtype=np.float64)[:, None]
        b = np.array(case["bias"], dtype=np.float64)[:, None]
        y = orc.hca_compress(x, g, b)
        assert y.shape == (len(case["x"]) // 128, 1)
        np.testing.assert_allclose(y[:, 0], case["y"], rtol=1e-13)
