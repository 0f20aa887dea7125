"""Pins for the oracle's four steps: compressor, indexer, top-512 transform,
sparse attention with the window.

Pages: 'Token 的一生：DSV4 架构与 DSpark' §1, §2.1, §2.2, §3.2 and
'DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）', section 'Compressed Sparse Attention
（CSA）'.  Pins: one-hot gates copy a row, equal logits with zero bias give the
mean, floor(L/4) output rows; the indexer against hand-worked values, a
library matmul on a single head and rotation invariance; the top-k against a
brute-force full sort; attention against torch's scaled-dot-product attention
in float64 and the k >= c4_len reduction to dense attention.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ compressor

def test_compress_golden(orc):
    for case in _gold("compress_example.json")["cases"]:
        T = len(case["x"])
        x = np.array(case["x"], dtype=np.float64)[:, None]
        g = np.array(case["gate"], dtype=np.float64)[:, None]
        b = np.array(case["bias"], dtype=np.float64)[:, None]
        y = orc.c4_compress(x, g, b)
        assert y.shape == (T // 4, 1)
        assert np.allclose(y[:, 0], case["y"], rtol=1e-14)


@pytest.mark.parametrize("T", [0, 1, 3, 4, 5, 7, 8, 9, 4095, 4096, 4097])
def test_compress_length_is_floor(orc, T):
    rng = np.random.default_rng(T)
    D = 8
    y = orc.c4_compress(rng.standard_normal((T, D)), rng.standard_normal((T, D)),
                        rng.standard_normal((4, D)))
    assert y.shape == (T // 4, D)
    assert orc.c4_len(T) == T // 4


def test_compress_one_hot_gate_copies_row(orc):
    rng = np.random.default_rng(0)
    T, D = 64, 576
    x = rng.standard_normal((T, D))
    pick = rng.integers(0, 4, size=T // 4)
    g = np.full((T, D), -300.0)
    for j, i in enumerate(pick):
        g[4 * j + i] = 300.0
    y = orc.c4_compress(x, g, np.zeros((4, D)))
    assert np.array_equal(y, x[4 * np.arange(T // 4) + pick])


def test_compress_bias_indexes_position_in_block(orc):
    rng = np.random.default_rng(1)
    T, D = 32, 16
    x = rng.standard_normal((T, D))
    for i in range(4):
        b = np.full((4, D), -400.0)
        b[i] = 400.0
        y = orc.c4_compress(x, np.zeros((T, D)), b)
        assert np.array_equal(y, x[i::4])


def test_compress_equal_logits_zero_bias_is_mean(orc):
    rng = np.random.default_rng(2)
    T, D = 40, 64
    x = rng.standard_normal((T, D))
    g = np.repeat(rng.standard_normal((T // 4, D)), 4, axis=0)   # equal within a block
    y = orc.c4_compress(x, g, np.zeros((4, D)))
    assert np.allclose(y, x.reshape(T // 4, 4, D).mean(1), rtol=1e-14, atol=1e-15)


def test_compress_weights_sum_to_one(orc):
    rng = np.random.default_rng(3)
    T, D = 16, 32
    c = rng.standard_normal(D)
    y = orc.c4_compress(np.tile(c, (T, 1)), rng.standard_normal((T, D)) * 5,
                        rng.standard_normal((4, D)))
    assert np.allclose(y, c, rtol=1e-13, atol=1e-14)


def test_compress_is_softmax_weighted_sum(orc):
    rng = np.random.default_rng(4)
    T, D = 12, 5
    x, g, b = rng.standard_normal((T, D)), rng.standard_normal((T, D)), rng.standard_normal((4, D))
    y = orc.c4_compress(x, g, b)
    a = scipy.special.softmax(g.reshape(3, 4, D) + b[None], axis=1)
    assert np.allclose(y, (a * x.reshape(3, 4, D)).sum(1), rtol=1e-13)


# ------------------------------------------------------------------ indexer

def test_indexer_golden(orc):
    g = _gold("indexer_example.json")
    q = np.array(g["q"], dtype=np.float64)[None]
    w = np.array(g["w"], dtype=np.float64)[None]
    k = np.array(g["k"], dtype=np.float64)
    out = orc.indexer_logits(q, w, k, [k.shape[0]])
    assert out[0].tolist() == g["logits"]


def test_indexer_single_head_is_relu_matmul(orc):
    rng = np.random.default_rng(5)
    q = rng.standard_normal((3, 1, 64))
    k = rng.standard_normal((300, 64))
    w = np.ones((3, 1))
    out = orc.indexer_logits(q, w, k, [300] * 3)
    ref = np.maximum(np.matmul(q[:, 0, :], k.T), 0.0)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_indexer_linear_in_weights_and_visibility(orc):
    rng = np.random.default_rng(6)
    q = rng.standard_normal((2, 8, 64))
    k = rng.standard_normal((100, 64))
    w = rng.uniform(size=(2, 8))
    a = orc.indexer_logits(q, w, k, [100, 37])
    b = orc.indexer_logits(q, 2 * w, k, [100, 37])
    assert np.allclose(b[0], 2 * a[0], rtol=1e-13)
    assert np.isnan(a[1, 37:]).all() and not np.isnan(a[1, :37]).any()
    per_head = [orc.indexer_logits(q[:, h:h + 1], w[:, h:h + 1], k, [100, 100]) for h in range(8)]
    assert np.allclose(sum(per_head)[0], a[0], rtol=1e-12)


def test_indexer_invariant_under_rotation(orc):
    rng = np.random.default_rng(7)
    for n in (64, 128):
        q = rng.standard_normal((4, 16, n))
        k = rng.standard_normal((200, n))
        w = rng.uniform(size=(4, 16))
        a = orc.indexer_logits(q, w, k, [200] * 4)
        b = orc.indexer_logits(orc.hadamard_rotate(q), w, orc.hadamard_rotate(k), [200] * 4)
        assert np.allclose(a, b, rtol=1e-10, atol=1e-10)


# ------------------------------------------------------------------ top-k

def _brute_topk(lg, n_vis, k):
    order = sorted(range(n_vis), key=lambda i: (-float(lg[i]), i))[:k]
    return sorted(order)


def test_topk_golden(orc):
    g = _gold("topk_example.json")
    lg = np.array(g["logits"], dtype=np.float32)
    phys, logical = orc.topk_transform(lg, len(lg), np.array(g["page_table"]), 100,
                                       k=g["k"], c4_page_size=g["c4_page_size"])
    assert logical.tolist() == g["logical"] and phys.tolist() == g["physical"]
    phys, logical = orc.topk_transform(lg, 3, np.array(g["page_table"]), 100,
                                       k=g["k"], c4_page_size=g["c4_page_size"])
    assert logical.tolist() == g["n_vis_3"]["logical"]
    assert phys.tolist() == g["n_vis_3"]["physical"]


@pytest.mark.parametrize("n", [0, 1, 2, 511, 512, 513, 1000, 5000])
def test_topk_matches_full_sort(orc, n):
    rng = np.random.default_rng(n)
    lg = np.round(rng.standard_normal(max(n, 1)) * 4).astype(np.float32)[:n]  # many ties
    if n > 3:
        lg[1] = -0.0
        lg[2] = 0.0
        lg[3] = -np.inf
    pages = (n + 63) // 64 + 1
    pt = rng.permutation(pages + 3).astype(np.int32)[:pages]
    phys, logical = orc.topk_transform(lg, n, pt, (pages + 3) * 64)
    want = _brute_topk(lg, n, 512)
    m = len(want)
    assert logical[:m].tolist() == want
    assert (logical[m:] == -1).all() and (phys[m:] == -1).all()
    lgc = np.asarray(want, dtype=np.int64)
    assert np.array_equal(phys[:m], pt[lgc // 64].astype(np.int64) * 64 + lgc % 64)


def test_topk_all_equal_and_identity_pages(orc):
    lg = np.full(3000, 1.5, dtype=np.float32)
    pt = np.arange(47, dtype=np.int32)
    phys, logical = orc.topk_transform(lg, 3000, pt, 47 * 64)
    assert logical.tolist() == list(range(512))
    assert phys.tolist() == list(range(512))


def test_topk_rejects_bad_page(orc):
    lg = np.arange(100, dtype=np.float32)
    with pytest.raises(IndexError):
        orc.topk_transform(lg, 100, np.array([0, 5], dtype=np.int32), 64 * 5)


# ------------------------------------------------------------------ attention

def test_attention_golden(orc):
    g = _gold("attention_example.json")
    q = np.zeros((1, 576))
    for d, v in g["q_nonzero"]:
        q[0, d] = v
    rows = np.zeros((2, 576))
    for r, nz in enumerate(g["rows_nonzero"]):
        for d, v in nz:
            rows[r, d] = v
    out, lse = orc.sparse_attention(q, rows, 1.0)
    want = np.zeros(512)
    for d, v in g["out_nonzero"]:
        want[d] = v
    assert np.allclose(out[0], want, rtol=1e-14, atol=1e-15)
    assert math.isclose(lse[0], g["lse"], rel_tol=1e-14)


def test_attention_matches_sdpa(orc):
    rng = np.random.default_rng(8)
    H, R = 16, 300
    q = rng.standard_normal((H, 576))
    rows = rng.standard_normal((R, 576))
    tau = 1 / math.sqrt(576)
    out, lse = orc.sparse_attention(q, rows, tau)
    tq = torch.tensor(q)[None, :, None, :]                          # [1, H, 1, 576]
    tk = torch.tensor(rows)[None, None].expand(1, H, R, 576)
    tv = torch.tensor(rows[:, :512])[None, None].expand(1, H, R, 512)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=tau)[0, :, 0]
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-13)
    z = tau * q @ rows.T
    assert np.allclose(lse, scipy.special.logsumexp(z, axis=1), rtol=1e-13)


def test_attention_single_row_and_uniform(orc):
    rng = np.random.default_rng(9)
    rows = rng.standard_normal((1, 576))
    out, _ = orc.sparse_attention(rng.standard_normal((4, 576)), rows, 0.3)
    assert np.allclose(out, np.tile(rows[0, :512], (4, 1)), rtol=1e-14)
    rows = rng.standard_normal((77, 576))
    out, lse = orc.sparse_attention(np.zeros((2, 576)), rows, 0.3)
    assert np.allclose(out, np.tile(rows[:, :512].mean(0), (2, 1)), rtol=1e-12)
    assert np.allclose(lse, math.log(77))
    out, lse = orc.sparse_attention(np.ones((1, 576)), np.zeros((0, 576)), 1.0)
    assert (out == 0).all() and np.isneginf(lse).all()


def test_topk_then_attention_equals_dense_when_k_covers_all(orc):
    """With n_c4 <= 512 every compressed row is selected, so the sparse path is
    dense attention over all compressed rows plus the window (brute force)."""
    rng = np.random.default_rng(10)
    L, W, H, Hi, Di = 1500, 128, 4, 8, 64       # n_c4 = 375 <= 512
    n_c4 = orc.c4_len(L)
    c4_rows = rng.standard_normal((n_c4, 576))
    raw_rows = rng.standard_normal((L, 576))
    qi, w = rng.standard_normal((1, Hi, Di)), rng.uniform(size=(1, Hi))
    k = rng.standard_normal((n_c4, Di))
    lg = orc.indexer_logits(qi, w, k, [n_c4])[0]
    pt = np.arange(8, dtype=np.int32)
    phys, logical = orc.topk_transform(lg, n_c4, pt, 8 * 64)
    assert sorted(logical[logical >= 0].tolist()) == list(range(n_c4))
    pos = L - 1
    win = orc.window_positions(pos, W)
    q = rng.standard_normal((H, 576))
    sel = np.concatenate([c4_rows[logical[logical >= 0]], raw_rows[win]])
    out, _ = orc.sparse_attention(q, sel, 0.05)
    dense = np.concatenate([c4_rows, raw_rows[pos - W + 1:pos + 1]])
    tq = torch.tensor(q)[None, :, None, :]
    tk = torch.tensor(dense)[None, None].expand(1, H, -1, 576)
    tv = torch.tensor(dense[:, :512])[None, None].expand(1, H, -1, 512)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.05)[0, :, 0]
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_window_and_visibility_rules(orc):
    assert orc.window_positions(5, 128).tolist() == list(range(6))
    assert orc.window_positions(1000, 128).tolist() == list(range(873, 1001))
    # decode: a query at the last position L-1 sees floor(L/4) compressed rows
    for L in range(1, 40):
        assert orc.n_visible(L - 1) == orc.c4_len(L)
    assert [orc.n_visible(p) for p in range(9)] == [0, 0, 0, 1, 1, 1, 1, 2, 2]


def test_kv_row_codec(orc):
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((20, 576)) * 3).astype(np.float32).astype(np.float64)
    x[4, :128] = 0.0
    b8 = orc.kv_encode_rows(x, fp8=True)
    assert b8.shape == (20, 656)
    d8 = orc.kv_decode_rows(b8, fp8=True)
    s = b8[:, 512:528].copy().view(np.float32)
    amax = np.abs(x[:, :512].astype(np.float32)).reshape(20, 4, 128).max(2)
    assert np.array_equal(s[amax > 0], (amax / np.float32(448.0))[amax > 0])
    assert s[4, 0] == 1.0
    assert (np.abs(d8[:, :512] - x[:, :512]) <= np.abs(x[:, :512]) * 2.0 ** -4 +
            np.repeat(s, 128, axis=1) * 2.0 ** -10 + 1e-12).all()
    # the RoPE part is bf16 RNE in both formats
    assert np.array_equal(d8[:, 512:], torch.tensor(x[:, 512:]).float().bfloat16().double().numpy())
    b16 = orc.kv_encode_rows(x, fp8=False)
    d16 = orc.kv_decode_rows(b16, fp8=False)
    assert np.array_equal(d16, torch.tensor(x).float().bfloat16().double().numpy())


def test_step_query_filter_matches_the_full_step(orc):
    # computing only some query rows of a request gives those rows unchanged
    import os
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
    from compressed_sparse_attention_12_b200 import synth
    w = synth.workload("prefill", 1 / 64)
    d = synth.draw(w, "cpu")
    pt = synth.page_table(w)
    full = orc.step(w, d, pt)
    part = orc.step(w, d, pt, queries={0, 5, w.num_q - 1})
    assert sorted(part) == [0, 5, w.num_q - 1]
    for t, r in part.items():
        assert np.array_equal(r["logical"], full[t]["logical"])
        assert np.array_equal(r["logits"], full[t]["logits"])
        assert np.array_equal(r["out"], full[t]["out"])
