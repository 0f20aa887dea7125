"""HCA branch ("DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", section "Heavily
Compressed Attention（HCA）") on the GPU against the oracle: the 128-row
compressor (bf16 and FP8 rows, ragged requests, partial trailing blocks) and the
dense attention over every visible compressed row plus the raw window (decode
and prefill, FP8 and bf16 rows, 16 and 64 heads, requests with no complete
block, window 0)."""
import math

import numpy as np
import pytest
import torch

from gpu_util import bf16_bound, dev
from oracle import oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    from compressed_sparse_attention_12_b200 import build, csa
    build.build()
    return csa.lib()


def _csa():
    from compressed_sparse_attention_12_b200 import csa
    return csa


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _page_table(rng, bs, pages):
    perm = rng.permutation(bs * pages + 3).astype(np.int32)
    return perm[: bs * pages].reshape(bs, pages).copy(), bs * pages + 3


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
def test_hca_compress(fmt):
    csa = _csa()
    rng = np.random.default_rng(11)
    new = np.array([3 * 128 + 50, 128, 0, 300, 127], dtype=np.int64)
    start = np.array([0, 128 * 7, 256, 128 * 40, 0], dtype=np.int64)
    bs = len(new)
    cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    x = rng.standard_normal((int(new.sum()), 576)).astype(np.float32)
    gate = rng.standard_normal((int(new.sum()), 576)).astype(np.float32)
    bias = (rng.standard_normal((128, 576)) * 0.1).astype(np.float32)
    pages = 64
    pt, n_pages = _page_table(rng, bs, pages)
    n_slots = n_pages * 2
    rb = csa.csa_kv_row_bytes(1 if fmt == "fp8" else 0)
    cache = torch.full((n_slots, rb), 0xCD, dtype=torch.uint8, device="cuda")
    st = _status()
    kind = csa.CSA_OUT_KV_FP8 if fmt == "fp8" else csa.CSA_OUT_KV_BF16
    csa.csa_hca_compress(dev(x), dev(gate), dev(bias), dev(cu), dev(start.astype(np.int32)),
                         int(new.max()), dev(pt), kind, cache, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = cache.cpu().numpy()
    written = np.zeros(n_slots, dtype=bool)
    for b in range(bs):
        xb, gb = x[cu[b]:cu[b + 1]].astype(np.float64), gate[cu[b]:cu[b + 1]].astype(np.float64)
        y = orc.hca_compress(xb, gb, bias.astype(np.float64))
        assert y.shape[0] == new[b] // 128
        for i in range(y.shape[0]):
            j = start[b] // 128 + i
            slot = pt[b, j // 2] * 2 + j % 2
            written[slot] = True
            gr = orc.kv_decode_rows(got[slot], fmt == "fp8")[0]
            blk = np.abs(xb[128 * i:128 * i + 128]).max(0)
            if fmt == "bf16":
                assert (np.abs(gr - y[i]) <= bf16_bound(y[i], floor=1e-6 * blk)).all()
            else:
                s = got[slot, 512:528].copy().view(np.float32).astype(np.float64)
                rs = orc.kv_encode_rows(y[i:i + 1], True)[0][512:528].copy().view(np.float32)
                assert np.allclose(s, rs.astype(np.float64), rtol=1e-5)
                bound = 2.0 ** -3 * np.abs(y[i, :512]) + np.repeat(s, 128) * 2.0 ** -9
                assert (np.abs(gr[:512] - y[i, :512]) <= bound).all()
                assert (np.abs(gr[512:] - y[i, 512:]) <=
                        bf16_bound(y[i, 512:], floor=1e-6 * blk[512:])).all()
    assert written.sum() == sum(n // 128 for n in new)
    assert (got[~written] == 0xCD).all()


def test_hca_compress_rejects_misaligned_start():
    csa = _csa()
    rng = np.random.default_rng(12)
    x = rng.standard_normal((256, 576)).astype(np.float32)
    cu = np.array([0, 256], dtype=np.int32)
    pt = np.arange(8, dtype=np.int32)[None]
    cache = torch.zeros((16, 1152), dtype=torch.uint8, device="cuda")
    st = _status()
    csa.csa_hca_compress(dev(x), dev(x), dev(np.zeros((128, 576), np.float32)), dev(cu),
                         dev(np.array([64], np.int32)), 256, dev(pt), csa.CSA_OUT_KV_BF16, cache,
                         status=st)
    torch.cuda.synchronize()
    assert st.item() == csa.CSA_ERR_BOUNDS
    assert (cache.cpu().numpy() == 0).all()


def _hca_case(kv_fmt, heads, decode, window, seed):
    rng = np.random.default_rng(seed)
    fp8 = kv_fmt == "fp8"
    # request 0 has 1562 HCA rows: with the window, more than one split's worth
    # of tiles, so prefill splits too
    L = np.array([200_000, 100, 128 * 40 + 7, 5000], dtype=np.int64)
    bs = len(L)
    q_lens = np.array([1, 1, 1, 1]) if decode else np.array([3, 1, 40, 2])
    pages = int(max((L + 255) // 256))
    # shuffled page ids; the pages holding window rows get the 16 smallest ids
    # so that the raw cache only needs those 16 pages
    n_pages = bs * pages + 16
    pt = rng.permutation(np.arange(16, n_pages)).astype(np.int32)[: bs * pages].reshape(bs, pages)
    small = 0
    for b in range(bs):
        lo = max(0, int(L[b] - q_lens[b]) - window + 1)
        for pg in range(lo // 256, (int(L[b]) - 1) // 256 + 1):
            pt[b, pg] = small
            small += 1
    assert small <= 16
    rb = 656 if fp8 else 1152
    hca_cache = np.zeros((n_pages * 2, rb), dtype=np.uint8)
    raw_cache = np.zeros((16 * 256, rb), dtype=np.uint8)
    hrows, rrows = {}, {}
    for b in range(bs):
        n = int(L[b] // 128)
        rows = rng.standard_normal((n, 576)) * (1 + (b == 2))
        enc = orc.kv_encode_rows(rows, fp8) if n else np.zeros((0, rb), np.uint8)
        s = np.arange(n)
        hca_cache[pt[b, s // 2].astype(np.int64) * 2 + s % 2] = enc
        hrows[b] = orc.kv_decode_rows(enc, fp8) if n else np.zeros((0, 576))
        lo = max(0, int(L[b] - q_lens[b]) - window + 1)
        pos = np.arange(lo, L[b])
        rr = rng.standard_normal((len(pos), 576))
        renc = orc.kv_encode_rows(rr, fp8)
        raw_cache[pt[b, pos // 256].astype(np.int64) * 256 + pos % 256] = renc
        rrows[b] = dict(zip(pos.tolist(), orc.kv_decode_rows(renc, fp8)))
    nq = int(q_lens.sum())
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q_pos = np.concatenate([np.arange(L[b] - q_lens[b], L[b]) for b in range(bs)]).astype(np.int32)
    q = torch.randn((nq, heads, 576), generator=torch.Generator().manual_seed(seed)).bfloat16()
    return dict(L=L, pt=pt, hca=hca_cache, raw=raw_cache, hrows=hrows, rrows=rrows, cu_q=cu_q,
                q_pos=q_pos, q=q, nq=nq)


@pytest.mark.parametrize("kv_fmt,heads,decode,window", [("fp8", 64, True, 128),
                                                        ("bf16", 16, True, 128),
                                                        ("fp8", 64, False, 128),
                                                        ("bf16", 64, False, 0),
                                                        ("fp8", 16, True, 0)])
def test_hca_attention(kv_fmt, heads, decode, window):
    csa = _csa()
    c = _hca_case(kv_fmt, heads, decode, window, seed=heads + window + decode)
    max_hca = int(max(c["L"]) // 128)
    out = torch.empty((c["nq"], heads, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((c["nq"], heads), dtype=torch.float32, device="cuda")
    st = _status()
    sm = 1.0 / math.sqrt(576)
    csa.csa_hca_attention(c["q"].cuda(), dev(c["hca"]), dev(c["raw"]), 1 if kv_fmt == "fp8" else 0,
                          dev(c["pt"]), dev(c["L"].astype(np.int32)), dev(c["cu_q"]),
                          dev(c["q_pos"]), max_hca, window, sm, decode, out, lse, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    go = out.float().cpu().numpy()
    gl = lse.cpu().numpy()
    tol = 2e-2 if kv_fmt == "fp8" else 5e-3
    qf = c["q"].double().numpy()
    for t in range(c["nq"]):
        b = int(np.searchsorted(c["cu_q"], t, side="right") - 1)
        p = int(c["q_pos"][t])
        nv = min(int(c["L"][b] // 128), orc.hca_visible(p))
        win = orc.window_positions(p, window)
        wrows = np.array([c["rrows"][b][int(r)] for r in win]).reshape(-1, 576)
        if nv + len(wrows) == 0:
            continue
        ro, rl = orc.hca_attention(qf[t], c["hrows"][b][:nv], wrows, sm)
        err = np.abs(go[t] - ro) - bf16_bound(ro, rel=0.0)
        assert err.max() <= tol, (t, err.max())
        assert np.abs(gl[t] - rl).max() <= 2e-2, t


def test_hca_attention_too_long_is_unsupported():
    csa = _csa()
    c = _hca_case("bf16", 16, True, 128, seed=3)
    out = torch.empty((c["nq"], 16, 512), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(csa.CsaError) as e:
        csa.csa_hca_attention(c["q"].cuda(), dev(c["hca"]), dev(c["raw"]), 0, dev(c["pt"]),
                              dev(c["L"].astype(np.int32)), dev(c["cu_q"]), dev(c["q_pos"]),
                              csa.HCA_MAX_ROWS, 128, 0.04, True, out)
    assert e.value.code == csa.CSA_ERR_UNSUPPORTED


def _hca_step_check(name, scale, sample=None):
    """A whole HCA-layer step (compressor + dense attention) through HcaBatch, in
    the benchmark's launch shapes, against oracle.hca_step on the same drawn
    buffers (each side encodes its own caches)."""
    from compressed_sparse_attention_12_b200 import pipeline, synth
    w = synth.workload(name, scale)
    data = synth.draw_hca(w, "cuda")
    batch = pipeline.HcaBatch(w, data)
    batch.step()
    torch.cuda.synchronize()
    batch.check_status()
    reqs = None
    if sample is not None:
        reqs = sorted(set(int(np.searchsorted(w.cu_q, t, side="right") - 1) for t in sample))
    ref = orc.hca_step(w, data, batch.pt_host, requests=reqs, sm_scale=batch.sm_scale)
    go = batch.out.float().cpu().numpy()
    gl = batch.lse.cpu().numpy()
    tol = 2e-2 if w.kv_fmt == "fp8" else 5e-3
    rows = sample if sample is not None else sorted(ref)
    assert rows
    for t in rows:
        r = ref[t]
        err = np.abs(go[t] - r["out"]) - bf16_bound(r["out"], rel=0.0)
        assert err.max() <= tol, (t, err.max())
        assert np.abs(gl[t] - r["lse"]).max() <= 2e-2, t
    return w, ref


@pytest.mark.parametrize("name,scale", [("hca_128k", 1 / 64), ("hca_1m", 1 / 64),
                                        ("hca_prefill", 1 / 16)])
def test_hca_step_end_to_end(name, scale):
    w, ref = _hca_step_check(name, scale)
    # the step's compressor wrote at least one of the rows attended to
    from compressed_sparse_attention_12_b200 import synth
    assert synth.hca_plan(w)[1].sum() > 0


def test_hca_full_size_decode_128k():
    _hca_step_check("hca_128k", 1.0)


def test_hca_full_size_decode_1m():
    _hca_step_check("hca_1m", 1.0)


def test_hca_full_size_prefill_sampled():
    # first, a middle and the last query tokens of the 4096-token prefill
    _hca_step_check("hca_prefill", 1.0, sample=[0, 1, 127, 2047, 4094, 4095])
