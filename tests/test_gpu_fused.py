"""The fused indexer + top-512 (csa_indexer_topk512, and its two halves
csa_indexer_select + csa_topk512_merge) against the separate calls
(csa_indexer_logits then csa_topk512_page_transform) on the same inputs:
logits, physical and raw indices must agree bit for bit.  The separate calls
are themselves checked against the oracle in test_gpu_steps.py and
test_gpu_pipeline.py; the fused path changes where the chunk selection runs,
not what it computes.  Shapes span one-chunk rows, rows below 512 keys,
causal multi-query rows (prefill, ragged), the 8-row 262144-key rows of the
1M decode and the full 32 x 32768 decode batch."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    from compressed_sparse_attention_12_b200 import build, csa
    build.build()
    return csa.lib()


def _batch(name, scale, paged=False):
    from compressed_sparse_attention_12_b200 import pipeline, synth
    w = synth.workload(name, scale)
    data = synth.draw(w, "cuda")
    return w, pipeline.CsaBatch(w, data, paged_fp4=paged)


def _separate(batch):
    batch.logits.fill_(float("nan"))
    batch.index()
    batch.select()
    torch.cuda.synchronize()
    batch.check_status()
    return batch.logits.clone(), batch.indices.clone(), batch.raw_indices.clone()


@pytest.mark.parametrize("name,scale,paged", [("tiny", 1.0, False), ("decode_128k", 1 / 64, False),
                                              ("decode_128k", 1.0, False), ("decode_1m", 1.0, False),
                                              ("decode_1m_wide", 1 / 16, False),
                                              ("ragged", 1 / 32, False), ("prefill", 1 / 16, False),
                                              ("decode_1m_wide", 1 / 16, True)])
def test_fused_equals_separate(name, scale, paged):
    w, batch = _batch(name, scale, paged)
    lg, idx, raw = _separate(batch)
    batch.logits.fill_(float("nan"))
    batch.indices.fill_(-7)
    batch.raw_indices.fill_(-7)
    batch.index_select()
    torch.cuda.synchronize()
    batch.check_status()
    n = batch.max_c4
    assert torch.equal(batch.logits[:, :n].isnan(), lg[:, :n].isnan())
    vis = ~lg[:, :n].isnan()
    assert torch.equal(batch.logits[:, :n][vis], lg[:, :n][vis])
    assert torch.equal(batch.indices, idx)
    assert torch.equal(batch.raw_indices, raw)


@pytest.mark.parametrize("name,scale", [("decode_128k", 1 / 16), ("ragged", 1 / 32)])
def test_select_then_merge_equals_fused(name, scale):
    from compressed_sparse_attention_12_b200 import csa
    w, batch = _batch(name, scale)
    batch.index_select()
    torch.cuda.synchronize()
    idx, raw = batch.indices.clone(), batch.raw_indices.clone()
    batch.indices.fill_(-7)
    batch.raw_indices.fill_(-7)
    ws = torch.empty_like(batch.fused_ws)
    csa.csa_indexer_select(batch.q_codes, batch.q_bsc, batch.w_fold, w.idx_heads, w.idx_dim,
                           batch.key_fmt, batch.k_codes, batch.k_bsc, batch.k_scales,
                           batch.page_table, batch.c4_lens, batch.cu_q, batch.q_pos, batch.max_c4,
                           batch.logits, ws, num_slots=batch.c4_slots_n, status=batch.status)
    csa.csa_topk512_merge(w.num_q, w.idx_heads, w.idx_dim, batch.key_fmt, batch.c4_lens,
                          batch.cu_q, batch.q_pos, batch.page_table, batch.c4_slots_n,
                          batch.max_c4, batch.indices, ws, raw_indices=batch.raw_indices,
                          status=batch.status)
    torch.cuda.synchronize()
    batch.check_status()
    assert torch.equal(batch.indices, idx)
    assert torch.equal(batch.raw_indices, raw)


def test_fused_workspace_is_checked():
    from compressed_sparse_attention_12_b200 import csa
    w, batch = _batch("decode_128k", 1 / 64)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(csa.CsaError) as e:
        csa.csa_indexer_topk512(batch.q_codes, batch.q_bsc, batch.w_fold, w.idx_heads,
                                w.idx_dim, batch.key_fmt, batch.k_codes, batch.k_bsc,
                                batch.k_scales, batch.page_table, batch.c4_lens, batch.cu_q,
                                batch.q_pos, batch.max_c4, batch.logits, batch.indices,
                                batch.raw_indices, small, status=batch.status)
    assert e.value.code == csa.CSA_ERR_WORKSPACE
