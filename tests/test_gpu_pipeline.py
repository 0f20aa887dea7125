"""End-to-end GPU runs of the whole CSA step against the oracle's whole step,
and parity at the full benchmark sizes in the benchmark's launch shapes.

End to end, each side quantises its own caches from the same drawn floats, so
the top-512 sets can differ where two logits sit within rounding of each
other; the set overlap is reported and must stay near 1, and queries whose
sets agree must match within the attention tolerance.  At full size the
indexer and top-512 are checked on oracle-quantised keys (bit-exact indices)
and the attention on sampled queries.
"""
import math

import numpy as np
import pytest
import torch

from gpu_util import bf16_bound, dev, index_arrays, rel_close
from oracle import oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    from compressed_sparse_attention_12_b200 import build, csa
    build.build()
    return csa.lib()


def _gpu(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


@pytest.mark.parametrize("name,scale,paged", [("tiny", 1.0, False), ("decode_128k", 1 / 64, False),
                                              ("decode_1m", 1 / 256, False),
                                              ("decode_1m_wide", 1 / 256, False),
                                              ("ragged", 1 / 128, False), ("prefill", 1 / 64, False),
                                              ("decode_1m", 1 / 256, True),
                                              ("ragged", 1 / 128, True)])
def test_step_end_to_end(name, scale, paged):
    """paged: FP4 index keys kept as CSA_FMT_FP4_PAGE records (the compressor
    writes them, the indexer reads them)."""
    from compressed_sparse_attention_12_b200 import pipeline, synth
    w = synth.workload(name, scale)
    data = synth.draw(w, "cpu")
    batch = pipeline.CsaBatch(w, _gpu(data), paged_fp4=paged)
    batch.step()
    torch.cuda.synchronize()
    batch.check_status()
    ref = orc.step(w, data, batch.pt_host, sm_scale=batch.sm_scale)
    raw = batch.raw_indices.cpu().numpy()
    phys = batch.indices.cpu().numpy()
    out = batch.out.float().cpu().numpy()
    tol = 2e-2 if w.kv_fmt == "fp8" else 5e-3
    overlaps, exact = [], 0
    for t, r in ref.items():
        want = set(r["logical"][r["logical"] >= 0].tolist())
        got = set(raw[t][raw[t] >= 0].tolist())
        assert len(got) == len(want) == min(512, r["n_vis"])
        overlaps.append(len(got & want) / max(1, len(want)))
        # raw and physical indices agree through the page table
        g = raw[t][raw[t] >= 0]
        b = int(np.searchsorted(w.cu_q, t, side="right") - 1)
        assert np.array_equal(phys[t][:len(g)], batch.pt_host[b, g // 64] * 64 + g % 64)
        if got == want:
            exact += 1
            assert (np.abs(out[t] - r["out"]) - bf16_bound(r["out"], rel=0.0)).max() <= tol, t
    print(f"\n{name}: mean top-512 overlap {np.mean(overlaps):.5f}, "
          f"min {np.min(overlaps):.5f}, identical sets {exact}/{len(ref)}")
    assert np.mean(overlaps) >= 0.98
    assert exact >= 0.5 * len(ref)
    # every query: the attention on exactly the rows the GPU selected and its
    # window, decoded from the GPU's own cache bytes, against the oracle's
    fp8 = w.kv_fmt == "fp8"
    c4c = batch.c4_cache.cpu().numpy()
    rwc = batch.raw_cache.cpu().numpy()
    qf = data["q"].double().numpy()
    for t in ref:
        b = int(np.searchsorted(w.cu_q, t, side="right") - 1)
        sel = phys[t][phys[t] >= 0]
        win = orc.window_positions(int(w.q_pos[t]), w.window)
        rsl = orc.raw_slot(batch.pt_host[b], win)
        rows = np.concatenate([orc.kv_decode_rows(c4c[sel], fp8).reshape(-1, 576),
                               orc.kv_decode_rows(rwc[rsl], fp8).reshape(-1, 576)])
        ro, _ = orc.sparse_attention(qf[t], rows, batch.sm_scale)
        assert (np.abs(out[t] - ro) - bf16_bound(ro, rel=0.0)).max() <= tol, t


def _full_index_check(name, sample_q):
    """Indexer + top-512 at full size on oracle-quantised keys, in the launch
    shapes the benchmark uses; attention on sampled queries."""
    from compressed_sparse_attention_12_b200 import csa, synth
    w = synth.workload(name)
    pt = synth.page_table(w)
    rng = np.random.default_rng(17)
    n = int(w.c4_lens[0])
    assert (w.c4_lens == n).all()
    bs, Hi, Di = w.bs, w.idx_heads, w.idx_dim
    keys = (rng.standard_t(3, (bs * n, Di)) if w.key_dist == "student_t3"
            else rng.standard_normal((bs * n, Di)))
    kq = orc.index_quantise(keys, w.idx_fmt)
    s = np.arange(n)
    slots = np.concatenate([pt[b, s // 64].astype(np.int64) * 64 + s % 64 for b in range(bs)])
    n_slots = w.num_pages * 64
    kfmt = w.idx_fmt
    kc, kb, ks = index_arrays(kq, kfmt, Di, n_slots, slots)
    qx = rng.standard_normal((bs, Hi, Di))
    qq = orc.index_quantise(qx, w.idx_fmt)
    qc, qb, qs = index_arrays(qq, w.idx_fmt, Di, bs * Hi)
    ww = rng.uniform(size=(bs, Hi)).astype(np.float32)
    wf = (ww * (qq["scales"].reshape(bs, Hi) if w.idx_fmt != "bf16" else 1.0)).astype(np.float32)
    stride = (n + 15) // 16 * 16
    logits = torch.empty((bs, stride), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    c4 = dev(w.c4_lens.astype(np.int32))
    cu_q = dev(w.cu_q)
    q_pos = dev(w.q_pos)
    fmt = csa.FMT[kfmt]
    csa.csa_indexer_logits(qc, qb, dev(wf), Hi, Di, fmt, kc, kb, ks, dev(pt), c4, cu_q, q_pos, n,
                           logits, num_slots=n_slots, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = logits.cpu().numpy()[:, :n]
    kd = kq["deq"]
    qd = qq["deq"].reshape(bs, Hi, Di)
    ref_lg = np.empty((bs, n), dtype=np.float64)
    for b in range(bs):
        ref_lg[b] = orc.indexer_logits(qd[b:b + 1], ww[b:b + 1], kd[b * n:(b + 1) * n], [n])[0]
        assert rel_close(got[b], ref_lg[b], 1e-2).all(), b
    # top-512 on the oracle's logits (rounded to float, the stored type): bit-exact
    lg32 = np.zeros((bs, stride), dtype=np.float32)
    lg32[:, :n] = ref_lg.astype(np.float32)
    out = torch.empty((bs, 512), dtype=torch.int32, device="cuda")
    raw = torch.empty((bs, 512), dtype=torch.int32, device="cuda")
    csa.csa_topk512_page_transform(dev(lg32), c4, cu_q, q_pos, dev(pt), n_slots, n, out, raw,
                                   status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    go, gr = out.cpu().numpy(), raw.cpu().numpy()
    for b in range(bs):
        phys, logical = orc.topk_transform(lg32[b], n, pt[b], n_slots)
        assert np.array_equal(gr[b], logical) and np.array_equal(go[b], phys), b
    # attention on sampled queries, oracle-encoded rows at the selected and window slots
    fp8 = w.kv_fmt == "fp8"
    rb = 656 if fp8 else 1152
    c4_cache = torch.zeros((n_slots, rb), dtype=torch.uint8, device="cuda")
    raw_cache = torch.zeros((w.num_pages * 256, rb), dtype=torch.uint8, device="cuda")
    q = torch.randn((bs, w.heads, 576), generator=torch.Generator().manual_seed(3)).bfloat16()
    sm_scale = 1.0 / math.sqrt(576)
    want = {}
    for b in sample_q:
        sel = gr[b][gr[b] >= 0]
        rows = rng.standard_normal((len(sel), 576))
        enc = orc.kv_encode_rows(rows, fp8)
        c4_cache[dev(go[b][:len(sel)].astype(np.int64))] = dev(enc)
        L = int(w.seq_lens[b])
        win = orc.window_positions(L - 1, w.window)
        rr = rng.standard_normal((len(win), 576))
        renc = orc.kv_encode_rows(rr, fp8)
        rsl = pt[b, win // 256].astype(np.int64) * 256 + win % 256
        raw_cache[dev(rsl)] = dev(renc)
        allrows = np.concatenate([orc.kv_decode_rows(enc, fp8), orc.kv_decode_rows(renc, fp8)])
        want[b] = orc.sparse_attention(q[b].double().numpy(), allrows, sm_scale)
    o = torch.empty((bs, w.heads, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((bs, w.heads), dtype=torch.float32, device="cuda")
    csa.csa_sparse_mqa_decode(q.cuda(), c4_cache, raw_cache, csa.FMT[w.kv_fmt], out, dev(pt),
                              dev(w.seq_lens.astype(np.int32)), cu_q, q_pos, w.window, sm_scale, o,
                              lse, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    go_ = o.float().cpu().numpy()
    tol = 2e-2 if fp8 else 5e-3
    for b, (ro, rl) in want.items():
        assert (np.abs(go_[b] - ro) - bf16_bound(ro, rel=0.0)).max() <= tol, b
        assert np.abs(lse.cpu().numpy()[b] - rl).max() <= 2e-2, b


def _full_ragged_check(name, sample_q):
    """Indexer + top-512 at full size for workloads with any mix of request
    lengths and query rows per request (the ragged serving batch: lengths up to
    1M, compressed lengths below 512 padded with -1, 1 or 5 query rows per
    request): logits on oracle-quantised keys to 1e-2 on every visible key of
    every query row, top-512 bit-exact (with -1 padding) on the oracle's
    logits in the benchmark's launch shape, attention on sampled queries."""
    from compressed_sparse_attention_12_b200 import csa, synth
    w = synth.workload(name)
    pt = synth.page_table(w)
    rng = np.random.default_rng(23)
    bs, Hi, Di, nq = w.bs, w.idx_heads, w.idx_dim, w.num_q
    c4 = w.c4_lens.astype(np.int64)
    off = np.concatenate([[0], np.cumsum(c4)])
    n_keys = int(off[-1])
    keys = (rng.standard_t(3, (n_keys, Di)) if w.key_dist == "student_t3"
            else rng.standard_normal((n_keys, Di)))
    kq = orc.index_quantise(keys, w.idx_fmt)
    del keys
    slots = np.concatenate([pt[b, np.arange(c4[b]) // 64].astype(np.int64) * 64 +
                            np.arange(c4[b]) % 64 for b in range(bs)])
    n_slots = w.num_pages * 64
    kfmt = w.idx_fmt
    kc, kb, ks = index_arrays(kq, kfmt, Di, n_slots, slots)
    qx = rng.standard_normal((nq, Hi, Di))
    qq = orc.index_quantise(qx, w.idx_fmt)
    qc, qb, qs = index_arrays(qq, w.idx_fmt, Di, nq * Hi)
    ww = rng.uniform(size=(nq, Hi)).astype(np.float32)
    wf = (ww * (qq["scales"].reshape(nq, Hi) if w.idx_fmt != "bf16" else 1.0)).astype(np.float32)
    max_c4 = int(c4.max())
    stride = (max_c4 + 15) // 16 * 16
    logits = torch.empty((nq, stride), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    c4_d, cu_q, q_pos = dev(c4.astype(np.int32)), dev(w.cu_q), dev(w.q_pos)
    csa.csa_indexer_logits(qc, qb, dev(wf), Hi, Di, csa.FMT[kfmt], kc, kb, ks, dev(pt), c4_d,
                           cu_q, q_pos, max_c4, logits, num_slots=n_slots, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = logits.cpu().numpy()
    kd = kq["deq"]
    qd = qq["deq"].reshape(nq, Hi, Di)
    lg32 = np.zeros((nq, stride), dtype=np.float32)
    nv = np.zeros(nq, dtype=np.int64)
    req = np.zeros(nq, dtype=np.int64)
    for b in range(bs):
        for t in range(int(w.cu_q[b]), int(w.cu_q[b + 1])):
            req[t] = b
            nv[t] = min(int(c4[b]), (int(w.q_pos[t]) + 1) // 4)
            if nv[t] == 0:
                continue
            ref = orc.indexer_logits(qd[t:t + 1], ww[t:t + 1], kd[off[b]:off[b] + c4[b]],
                                     [nv[t]])[0, :nv[t]]
            assert rel_close(got[t, :nv[t]], ref, 1e-2).all(), (b, t)
            lg32[t, :nv[t]] = ref.astype(np.float32)
    del kd
    out = torch.empty((nq, 512), dtype=torch.int32, device="cuda")
    raw = torch.empty((nq, 512), dtype=torch.int32, device="cuda")
    csa.csa_topk512_page_transform(dev(lg32), c4_d, cu_q, q_pos, dev(pt), n_slots, max_c4, out, raw,
                                   status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    go, gr = out.cpu().numpy(), raw.cpu().numpy()
    short = 0
    for t in range(nq):
        phys, logical = orc.topk_transform(lg32[t], int(nv[t]), pt[req[t]], n_slots)
        assert np.array_equal(gr[t], logical) and np.array_equal(go[t], phys), t
        short += int(nv[t] < 512)
    if name == "ragged":
        assert short > 0              # some rows are padded with -1
    # attention on sampled queries: rows drawn per slot (queries of one request
    # share the rows of the slots they both select)
    fp8 = w.kv_fmt == "fp8"
    rb = 656 if fp8 else 1152
    c4_cache = torch.zeros((n_slots, rb), dtype=torch.uint8, device="cuda")
    raw_cache = torch.zeros((w.num_pages * 256, rb), dtype=torch.uint8, device="cuda")
    q = torch.randn((nq, w.heads, 576), generator=torch.Generator().manual_seed(5)).bfloat16()
    sm_scale = 1.0 / math.sqrt(576)
    c4_rows, raw_rows = {}, {}

    def rows_at(table, cache, sl):
        new = [int(x) for x in sl if int(x) not in table]
        if new:
            enc = orc.kv_encode_rows(rng.standard_normal((len(new), 576)), fp8)
            cache[dev(np.asarray(new, dtype=np.int64))] = dev(enc)
            for x, e in zip(new, orc.kv_decode_rows(enc, fp8)):
                table[x] = e
        return np.array([table[int(x)] for x in sl]).reshape(-1, 576)

    want = {}
    for t in sample_q:
        b = int(req[t])
        sel = go[t][go[t] >= 0]
        win = orc.window_positions(int(w.q_pos[t]), w.window)
        rsl = pt[b, win // 256].astype(np.int64) * 256 + win % 256
        want[t] = (sel, rsl)
    for t, (sel, rsl) in want.items():
        rows_at(c4_rows, c4_cache, sel)
        rows_at(raw_rows, raw_cache, rsl)
    o = torch.empty((nq, w.heads, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((nq, w.heads), dtype=torch.float32, device="cuda")
    decode = bool((w.q_lens <= 8).all())
    fn = csa.csa_sparse_mqa_decode if decode else csa.csa_sparse_mqa_prefill
    fn(q.cuda(), c4_cache, raw_cache, csa.FMT[w.kv_fmt], out, dev(pt),
       dev(w.seq_lens.astype(np.int32)), cu_q, q_pos, w.window, sm_scale, o, lse, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    go_, gl = o.float().cpu().numpy(), lse.cpu().numpy()
    tol = 2e-2 if fp8 else 5e-3
    for t, (sel, rsl) in want.items():
        allrows = np.concatenate([rows_at(c4_rows, c4_cache, sel), rows_at(raw_rows, raw_cache, rsl)])
        ro, rl = orc.sparse_attention(q[t].double().numpy(), allrows, sm_scale)
        assert (np.abs(go_[t] - ro) - bf16_bound(ro, rel=0.0)).max() <= tol, t
        assert np.abs(gl[t] - rl).max() <= 2e-2, t


def test_full_size_decode_128k():
    _full_index_check("decode_128k", sample_q=[0, 13, 31])


def test_full_size_decode_1m():
    _full_index_check("decode_1m", sample_q=[0, 7])


def test_full_size_decode_1m_wide():
    _full_ragged_check("decode_1m_wide", sample_q=[0, 3, 7])


def test_full_size_ragged():
    # queries 0 and 1 belong to the two requests shorter than 512 compressed
    # rows; the last five are the verify rows of the last (5-row) request
    from compressed_sparse_attention_12_b200 import synth
    w = synth.workload("ragged")
    last = int(w.num_q)
    _full_ragged_check("ragged", sample_q=[0, 1, 2, 40, last - 5, last - 1])


def test_full_size_prefill_indexer_shared_codes():
    """The indexer in the prefill launch shape (one request, 4096 causal query
    rows seeing 65536-66560 keys, query rows grouped four to a tile column
    block) on keys and queries quantised by the oracle: sampled rows against
    the oracle's logits at 1e-2 relative, covering every row position inside a
    query group and both ends of the chunk."""
    from compressed_sparse_attention_12_b200 import csa, synth
    w = synth.workload("prefill")
    assert w.bs == 1
    pt = synth.page_table(w)
    rng = np.random.default_rng(29)
    n = int(w.c4_lens[0])
    nq, Hi, Di = int(w.num_q), w.idx_heads, w.idx_dim
    keys = rng.standard_normal((n, Di))
    kq = orc.index_quantise(keys, w.idx_fmt)
    s = np.arange(n)
    slots = pt[0, s // 64].astype(np.int64) * 64 + s % 64
    n_slots = w.num_pages * 64
    kfmt = w.idx_fmt
    kc, kb, ks = index_arrays(kq, kfmt, Di, n_slots, slots)
    qx = rng.standard_normal((nq, Hi, Di))
    qq = orc.index_quantise(qx, w.idx_fmt)
    qc, qb, qs = index_arrays(qq, w.idx_fmt, Di, nq * Hi)
    ww = rng.uniform(size=(nq, Hi)).astype(np.float32)
    wf = (ww * qq["scales"].reshape(nq, Hi)).astype(np.float32)
    stride = (n + 15) // 16 * 16
    logits = torch.full((nq, stride), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa.csa_indexer_logits(qc, qb, dev(wf), Hi, Di, csa.FMT[w.idx_fmt], kc, kb, ks, dev(pt),
                           dev(w.c4_lens.astype(np.int32)), dev(w.cu_q), dev(w.q_pos), n, logits,
                           status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    sample = [0, 1, 2, 3, 4, 5, 6, 7, 1029, 2046, 2047, 4092, 4093, 4094, 4095]
    got = logits[sample].cpu().numpy()
    kd = kq["deq"]
    qd = qq["deq"].reshape(nq, Hi, Di)
    for i, t in enumerate(sample):
        nv = min(n, orc.n_visible(int(w.q_pos[t])))
        assert 65536 <= nv <= n, (t, nv)
        ref = orc.indexer_logits(qd[t:t + 1], ww[t:t + 1], kd[:nv], [nv])[0]
        assert rel_close(got[i, :nv], ref, 1e-2).all(), t
        # keys past the causal limit are not written
        assert np.isnan(got[i, nv:]).all(), t


def test_full_size_prefill_sampled():
    """The 4096-token prefill on a 262144-token context at full size in the
    benchmark's separate form (plain indexer, two-stage top-k over rows of
    65536-66560 keys, per-query attention), against the oracle on sampled
    query rows: logits, top-512 bit-exact on the oracle's logits, attention
    where the selected sets agree."""
    from compressed_sparse_attention_12_b200 import csa, pipeline, synth
    w = synth.workload("prefill")
    data = synth.draw(w, "cuda")
    batch = pipeline.CsaBatch(w, data)
    batch.step(fused=False)
    torch.cuda.synchronize()
    batch.check_status()
    sample = [0, 1, 2047, 4094, 4095]
    ref = orc.step(w, data, batch.pt_host, queries=set(sample), sm_scale=batch.sm_scale)
    lg = batch.logits.cpu().numpy()
    raw = batch.raw_indices.cpu().numpy()
    out = batch.out.float().cpu().numpy()
    agree = 0
    for t in sample:
        r = ref[t]
        n = r["n_vis"]
        # each side quantises the index query and the keys pooled this step on
        # its own: a value on an FP8 rounding midpoint (float32 here, float64
        # there) takes the neighbouring code, which moves that query's logits
        # slightly (the share the quantiser and compressor tests allow); the
        # logits are checked exactly on shared codes in _full_index_check
        close = rel_close(lg[t, :n], r["logits"], 1e-2)
        assert close.mean() >= 0.99, (t, close.mean())
        assert rel_close(lg[t, :n], r["logits"], 5e-2).all(), t
        # top-512 on the oracle's float logits: bit-exact
        lg32 = np.zeros((1, batch.logit_stride), np.float32)
        lg32[0, :n] = r["logits"].astype(np.float32)
        o1 = torch.empty((1, 512), dtype=torch.int32, device="cuda")
        o2 = torch.empty((1, 512), dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        csa.csa_topk512_page_transform(dev(lg32), batch.c4_lens, dev(np.array([0, 1], np.int32)),
                                       batch.q_pos[t:t + 1], batch.page_table, batch.c4_slots_n,
                                       batch.max_c4, o1, o2, status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        p_ref, l_ref = orc.topk_transform(lg32[0], n, batch.pt_host[0], batch.c4_slots_n)
        assert np.array_equal(o2.cpu().numpy()[0], l_ref), t
        assert np.array_equal(o1.cpu().numpy()[0], p_ref), t
        want = set(r["logical"][r["logical"] >= 0].tolist())
        got = set(raw[t][raw[t] >= 0].tolist())
        assert len(got & want) / len(want) >= 0.98, t
        if got == want:
            agree += 1
            err = np.abs(out[t] - r["out"]) - bf16_bound(r["out"], rel=0.0)
            assert err.max() <= 2e-2, (t, err.max())
    assert agree >= 3
