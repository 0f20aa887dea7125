"""The algorithmic byte counts behind the benchmark's roofline figures,
against the closed forms of the workloads they describe."""
import os
import sys

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))

import bench  # noqa: E402
from compressed_sparse_attention_12_b200 import synth  # noqa: E402


def test_indexer_bytes_decode_128k():
    # 32 requests x 32768 keys of (128 FP8 codes + 4 B scale), plus 64 query
    # heads of (128 + 4) B codes and a 4 B weight per row; the 4 B logits are
    # counted apart
    w = synth.workload("decode_128k")
    assert bench.indexer_alg_bytes(w) == 32 * 32768 * 132 + 32 * 64 * (132 + 4)
    assert bench.indexer_logit_bytes(w) == 32 * 32768 * 4


def test_indexer_bytes_decode_1m_fp4():
    # FP4 8x64: a key is 32 code bytes + 4 block scales + a 4 B row scale
    w = synth.workload("decode_1m")
    assert bench.index_bytes_per_key(w) == 40
    assert bench.indexer_alg_bytes(w) == 8 * 262144 * 40 + 8 * 8 * (40 + 4)


def test_indexer_bytes_dsa_counts_every_raw_key():
    # ratio 1: query at position L-1 sees L keys
    w = synth.workload("dsa_128k")
    assert bench.indexer_alg_bytes(w, 1) == 32 * 131072 * 132 + 32 * 64 * (132 + 4)
    assert bench.indexer_logit_bytes(w, 1) == 32 * 131072 * 4


def test_step_bytes_decode_128k():
    # keys once, q codes + weights, 512 selected + 128 window rows of 656 B,
    # attention q (576 bf16) and out (512 bf16) per head
    w = synth.workload("decode_128k")
    want = (32 * 32768 * 132 + 32 * 64 * (132 + 4) + 32 * 640 * 656 +
            32 * 64 * (576 + 512) * 2)
    assert bench.step_alg_bytes(w) == want


def test_hca_attention_bytes():
    # every HCA row (131072/128 = 1024) and 128 window rows per query, plus q,
    # out and lse per head
    w = synth.workload("hca_128k")
    assert bench.hca_attn_alg_bytes(w) == 32 * (1024 + 128) * 656 + 32 * 64 * (1152 + 1024 + 4)


def test_prefill_counts_each_key_once_and_is_tensor_bound():
    # 4096 queries of one request share its 66560 keys: bytes count them once,
    # flops count every (query, key) pair; the intensity is far above the ridge
    w = synth.workload("prefill")
    L = 262144 + 4096
    nv = sum(min(L // 4, (p + 1) // 4) for p in range(L - 4096, L))
    assert bench.indexer_flops(w) == nv * 64 * 128 * 2
    assert bench.indexer_alg_bytes(w) == (L // 4) * 132 + 4096 * 64 * 136
    assert bench.indexer_logit_bytes(w) == nv * 4
    line = bench.indexer_roofline(w, 7.8e-3, 6551.4, "measured", None)
    assert line["bound"] == "tensor" and line["unit"] == "TFLOP/s"
    assert abs(line["achieved"] - nv * 64 * 128 * 2 / 7.8e-3 / 1e12) < 1e-6
    assert line["frac"] == line["achieved"] / line["peak"]


def test_decode_roofline_is_hbm_bound():
    w = synth.workload("decode_128k")
    line = bench.indexer_roofline(w, 43.1e-6, 6551.4, "measured", 144419328)
    assert line["bound"] == "hbm" and line["unit"] == "GB/s"
    assert line["alg_bytes_per_launch"] == 32 * 32768 * 132 + 32 * 64 * 136
    assert line["logit_bytes_per_launch"] == 32 * 32768 * 4
    assert line["traffic"] == 144419328
    assert line["intensity_flop_per_byte"] < line["ridge_flop_per_byte"]


def test_pack_inputs_and_rebinding_keep_each_input_at_its_offset():
    # the step inputs move into one buffer (256-byte aligned views); binding
    # them to another buffer of the same size keeps names, shapes and offsets
    import torch

    class B:
        pass

    b = B()
    b.q = torch.arange(6, dtype=torch.float32).reshape(2, 3)
    b.w = torch.arange(5, dtype=torch.int32)
    b.out = torch.zeros(4)
    arena = bench.pack_inputs(b, ["q", "w", "missing"], "cpu")
    assert [e[0] for e in arena.input_layout] == ["q", "w"]
    assert [e[1] % 256 for e in arena.input_layout] == [0, 0]
    assert torch.equal(b.q, torch.arange(6, dtype=torch.float32).reshape(2, 3))
    assert b.q.data_ptr() == arena.data_ptr()
    other = arena.clone()
    out2 = torch.ones(4)
    bench.bind_inputs(b, other, arena.input_layout, out2)
    assert b.q.data_ptr() == other.data_ptr() and b.out is out2
    assert torch.equal(b.w, torch.arange(5, dtype=torch.int32))
    assert b.w.data_ptr() == other.data_ptr() + arena.input_layout[1][1]
