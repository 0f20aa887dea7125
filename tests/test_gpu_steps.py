"""GPU parity of each step of the CUDA path against the fp64 oracle.

Each test feeds the library (through its C ABI binding) and the oracle the
same inputs -- seeded draws, or codes the oracle itself produced -- and
compares element by element:
  - KV row store: bit-exact;
  - rotation + quantisation: codes bit-exact except where the float32 and
    float64 rotations straddle a rounding midpoint (share <= 1e-3, and then
    only by one step), scales to float32 rounding;
  - compressor: 2e-3 relative in bf16 (floor 2e-3 of the block's max |x|),
    FP8 rows within one quantisation step;
  - indexer logits: 1e-2 relative (floor 1e-3 of the row's max);
  - top-512 indices: bit-exact;
  - attention: max abs 2e-2 (FP8 KV) / 5e-3 (bf16 KV).
"""
import math

import numpy as np
import pytest
import torch

from gpu_util import bf16_bound, code_values, dev, index_arrays, rel_close
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

FMT = {"bf16": 0, "fp8": 1, "fp4": 2, "fp4p": 4}


@pytest.fixture(scope="module", autouse=True)
def lib():
    from compressed_sparse_attention_12_b200 import build, csa
    build.build()
    return csa.lib()


def _csa():
    from compressed_sparse_attention_12_b200 import csa
    return csa


def zstatus():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


# ------------------------------------------------------------------ KV rows

@pytest.mark.parametrize("fmt", ["fp8", "bf16"])
def test_kv_store_bit_exact(fmt):
    csa = _csa()
    g = torch.Generator().manual_seed(11)
    n, n_slots = 300, 1000
    x = torch.randn(n, 576, generator=g) * torch.exp(torch.randn(n, 1, generator=g))
    x[5, :128] = 0.0
    x[6, 128:256] *= 1e-30
    x[7, 0] = 1e4
    x[8, 3] = -0.0
    slots = torch.randperm(n_slots, generator=g)[:n].int()
    slots[3] = -1
    rb = csa.csa_kv_row_bytes(FMT[fmt])
    cache = torch.full((n_slots, rb), 0xAB, dtype=torch.uint8, device="cuda")
    st = zstatus()
    csa.csa_kv_store(x.cuda(), slots.cuda(), FMT[fmt], cache, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    want = orc.kv_encode_rows(x.double().numpy(), fmt == "fp8")
    got = cache.cpu().numpy()
    s = slots.numpy()
    v = s >= 0
    assert np.array_equal(got[s[v]], want[v])
    untouched = np.setdiff1d(np.arange(n_slots), s[v])
    assert (got[untouched] == 0xAB).all()
    # a slot beyond the cache is reported and skipped
    bad = torch.tensor([n_slots + 5], dtype=torch.int32, device="cuda")
    csa.csa_kv_store(x[:1].cuda(), bad, FMT[fmt], cache, status=st)
    torch.cuda.synchronize()
    assert st.item() == csa.CSA_ERR_BOUNDS
    assert np.array_equal(cache.cpu().numpy(), got)


# ------------------------------------------------------------------ rotation + quantisation

def _compare_codes(got_codes, got_bsc, got_sc, ref, fmt, dim, rows):
    gv = code_values(got_codes, fmt, dim).reshape(rows, dim)
    if fmt == "bf16":
        rv = ref["deq"].reshape(rows, dim)
    elif fmt == "fp8":
        rv = orc.e4m3_table()[ref["codes"].reshape(rows, dim)]
    else:
        rv = orc.e2m1_table()[ref["codes"].reshape(rows, dim)]
    mism = gv != rv
    share = mism.mean()
    assert share <= 1e-3, f"code mismatch share {share}"
    if mism.any():
        a, b = np.abs(gv[mism]), np.abs(rv[mism])
        step = {"bf16": 2.0 ** -7, "fp8": 2.0 ** -3, "fp4": 0.5}[fmt]
        assert (np.abs(gv[mism] - rv[mism]) <= step * np.maximum(np.maximum(a, b), 1.0) + 1e-30).all()
    if fmt != "bf16":
        assert np.allclose(np.asarray(got_sc).reshape(-1), ref["scales"].reshape(-1), rtol=2 ** -21,
                           atol=0)
    if fmt == "fp4":
        bm = np.asarray(got_bsc).reshape(-1) != ref["block_scales"].reshape(-1)
        assert bm.mean() <= 1e-3
    return share


@pytest.mark.parametrize("fmt", ["fp8", "fp4", "bf16"])
@pytest.mark.parametrize("dim", [64, 128])
@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_hadamard_quant(fmt, dim, xdt):
    csa = _csa()
    g = torch.Generator().manual_seed(dim * 7 + len(fmt) + len(xdt))
    rows = 3000
    x = torch.randn(rows, dim, generator=g)
    x[::7] *= 50.0
    x[1] = 0.0
    x[2] = torch.randn(dim, generator=g) ** 3
    x[4, 5] = 1e6
    if xdt == "bf16":
        x = x.bfloat16()
    w = torch.rand(rows, generator=g)
    cb = {"bf16": 2 * dim, "fp8": dim, "fp4": dim // 2}[fmt]
    codes = torch.empty((rows, cb), dtype=torch.uint8, device="cuda")
    bsc = torch.empty((rows, dim // 16), dtype=torch.uint8, device="cuda") if fmt == "fp4" else None
    sc = torch.empty(rows, dtype=torch.float32, device="cuda") if fmt != "bf16" else None
    wo = torch.empty(rows, dtype=torch.float32, device="cuda")
    st = zstatus()
    csa.csa_hadamard_quant(x.cuda(), FMT[fmt], codes, bsc, sc, w_in=w.cuda(), w_out=wo, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = orc.index_quantise(x.double().numpy(), fmt)
    _compare_codes(codes.cpu().numpy(), None if bsc is None else bsc.cpu().numpy(),
                   None if sc is None else sc.cpu().numpy(), ref, fmt, dim, rows)
    want_w = w.numpy() * (sc.cpu().numpy() if sc is not None else 1.0)
    assert np.array_equal(wo.cpu().numpy(), want_w.astype(np.float32))


def test_hadamard_quant_row_map_scatter():
    csa = _csa()
    g = torch.Generator().manual_seed(3)
    rows, dim, n_out = 500, 128, 2000
    x = torch.randn(rows, dim, generator=g)
    rmap = torch.randperm(n_out, generator=g)[:rows].int()
    rmap[0] = -1
    codes = torch.full((n_out, dim), 0x55, dtype=torch.uint8, device="cuda")
    sc = torch.full((n_out,), -1.0, dtype=torch.float32, device="cuda")
    st = zstatus()
    csa.csa_hadamard_quant(x.cuda(), FMT["fp8"], codes, None, sc, row_map=rmap.cuda(), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = orc.index_quantise(x.double().numpy(), "fp8")
    r = rmap.numpy()
    got = codes.cpu().numpy()
    v = r >= 0
    assert (got[r[v]] == ref["codes"][v]).mean() > 0.999
    untouched = np.setdiff1d(np.arange(n_out), r[v])
    assert (got[untouched] == 0x55).all() and (sc.cpu().numpy()[untouched] == -1.0).all()


@pytest.mark.parametrize("dim", [64, 128])
def test_hadamard_quant_fp4_page_records(dim):
    """Index keys quantised straight into paged records equal the plain FP4
    arrays of the same call laid out as records, byte for byte, and untouched
    slots stay as they were."""
    from gpu_util import fp4_page_unpack
    csa = _csa()
    g = torch.Generator().manual_seed(11 + dim)
    rows, pages = 700, 20
    n_slots = pages * 64
    x = torch.randn(rows, dim, generator=g) * 3.0
    rmap = torch.randperm(n_slots, generator=g)[:rows].int()
    w = torch.rand(rows, generator=g)
    codes = torch.zeros((n_slots, dim // 2), dtype=torch.uint8, device="cuda")
    bsc = torch.zeros((n_slots, dim // 16), dtype=torch.uint8, device="cuda")
    sc = torch.ones(n_slots, dtype=torch.float32, device="cuda")
    wo = torch.empty(rows, dtype=torch.float32, device="cuda")
    rec = torch.full((pages, csa.index_record_bytes(dim)), 0x5A, dtype=torch.uint8, device="cuda")
    wo2 = torch.empty(rows, dtype=torch.float32, device="cuda")
    st = zstatus()
    csa.csa_hadamard_quant(x.cuda(), FMT["fp4"], codes, bsc, sc, row_map=rmap.cuda(),
                           w_in=w.cuda(), w_out=wo, status=st)
    csa.csa_hadamard_quant(x.cuda(), FMT["fp4p"], rec, None, None, row_map=rmap.cuda(),
                           w_in=w.cuda(), w_out=wo2, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    pk, pb, ps = fp4_page_unpack(rec.cpu().numpy(), dim)
    r = rmap.numpy()
    assert np.array_equal(pk[r], codes.cpu().numpy()[r])
    assert np.array_equal(pb[r], bsc.cpu().numpy()[r])
    assert np.array_equal(ps[r].view(np.uint32), sc.cpu().numpy()[r].view(np.uint32))
    assert np.array_equal(wo.cpu().numpy(), wo2.cpu().numpy())
    untouched = np.setdiff1d(np.arange(n_slots), r)
    assert (pk[untouched] == 0x5A).all() and (pb[untouched] == 0x5A).all()


# ------------------------------------------------------------------ compressor

def _compress_setup(dim, seed, new=(4096, 7, 0, 13, 4, 64)):
    rng = np.random.default_rng(seed)
    bs = len(new)
    start = np.array([0, 1024, 40, 1300, 8, 4096], dtype=np.int64)[:bs]
    cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    T = int(cu[-1])
    x = rng.standard_normal((T, dim)).astype(np.float32)
    gate = rng.standard_normal((T, dim)).astype(np.float32)
    bias = (rng.standard_normal((4, dim)) * 0.1).astype(np.float32)
    last_j = (start + np.asarray(new)) // 4
    pages_needed = (last_j + 63) // 64 + 1
    stride = int(pages_needed.max())
    n_pages = int(pages_needed.sum()) + 3
    perm = rng.permutation(n_pages).astype(np.int32)
    pt = np.full((bs, stride), -1, dtype=np.int32)
    o = 0
    for b in range(bs):
        pt[b, :pages_needed[b]] = perm[o:o + pages_needed[b]]
        o += pages_needed[b]
    return x, gate, bias, cu, start, pt, n_pages * 64, np.asarray(new)


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
def test_c4_compress_kv(fmt):
    csa = _csa()
    x, gate, bias, cu, start, pt, n_slots, new = _compress_setup(576, 1)
    rb = csa.csa_kv_row_bytes(FMT[fmt])
    cache = torch.full((n_slots, rb), 0xCD, dtype=torch.uint8, device="cuda")
    st = zstatus()
    kind = csa.CSA_OUT_KV_FP8 if fmt == "fp8" else csa.CSA_OUT_KV_BF16
    csa.csa_c4_compress(dev(x), dev(gate), dev(bias), dev(cu), dev(start.astype(np.int32)),
                        int(new.max()), dev(pt), kind, cache, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = cache.cpu().numpy()
    written = np.zeros(n_slots, dtype=bool)
    rne_mismatch, n_el = 0, 0
    for b in range(len(new)):
        xb, gb = x[cu[b]:cu[b + 1]].astype(np.float64), gate[cu[b]:cu[b + 1]].astype(np.float64)
        y = orc.c4_compress(xb, gb, bias.astype(np.float64))
        for i in range(y.shape[0]):
            j = start[b] // 4 + i
            slot = pt[b, j // 64] * 64 + j % 64
            written[slot] = True
            gr = orc.kv_decode_rows(got[slot], fmt == "fp8")[0]
            blk = np.abs(xb[4 * i:4 * i + 4]).max(0)
            if fmt == "bf16":
                assert (np.abs(gr - y[i]) <= bf16_bound(y[i], floor=1e-6 * blk)).all()
                rne_mismatch += int((orc.kv_encode_rows(y[i:i + 1], False)[0] != got[slot]).sum())
                n_el += 1152
            else:
                s = got[slot, 512:528].copy().view(np.float32).astype(np.float64)
                ref_row = orc.kv_encode_rows(y[i:i + 1], True)[0]
                rs = ref_row[512:528].copy().view(np.float32).astype(np.float64)
                assert np.allclose(s, rs, rtol=1e-5)
                lat = np.abs(gr[:512] - y[i, :512])
                bound = 2.0 ** -3 * np.abs(y[i, :512]) + np.repeat(s, 128) * 2.0 ** -9
                assert (lat <= bound).all()
                assert (np.abs(gr[512:] - y[i, 512:]) <= bf16_bound(y[i, 512:],
                                                                   floor=1e-6 * blk[512:])).all()
    assert (got[~written] == 0xCD).all()
    # the single float32 rounding agrees with the oracle's bf16 rounding except
    # where float32 and float64 straddle a rounding midpoint
    assert rne_mismatch <= 1e-3 * max(n_el, 1)


def test_c4_compress_one_hot_gate_copies_rows():
    csa = _csa()
    x, gate, bias, cu, start, pt, n_slots, new = _compress_setup(576, 2, new=(64, 8))
    rng = np.random.default_rng(0)
    pick = rng.integers(0, 4, size=x.shape[0] // 4)
    gate[:] = -300.0
    for j, i in enumerate(pick):
        gate[4 * j + i] = 300.0
    bias[:] = 0.0
    cache = torch.zeros((n_slots, 1152), dtype=torch.uint8, device="cuda")
    csa.csa_c4_compress(dev(x), dev(gate), dev(bias), dev(cu), dev(start.astype(np.int32)), 64,
                        dev(pt), csa.CSA_OUT_KV_BF16, cache)
    torch.cuda.synchronize()
    got = cache.cpu().numpy()
    for b in range(2):
        for i in range((cu[b + 1] - cu[b]) // 4):
            j = start[b] // 4 + i
            slot = pt[b, j // 64] * 64 + j % 64
            src = x[cu[b] + 4 * i + pick[cu[b] // 4 + i]]
            assert np.array_equal(got[slot], orc.kv_encode_rows(src[None].astype(np.float64),
                                                                False)[0])


def test_c4_compress_rejects_misaligned_start():
    csa = _csa()
    x, gate, bias, cu, start, pt, n_slots, new = _compress_setup(576, 3, new=(8, 8))
    start = start.copy()
    start[1] = 1026
    cache = torch.zeros((n_slots, 656), dtype=torch.uint8, device="cuda")
    st = zstatus()
    csa.csa_c4_compress(dev(x), dev(gate), dev(bias), dev(cu), dev(start.astype(np.int32)), 8,
                        dev(pt), csa.CSA_OUT_KV_FP8, cache, status=st)
    torch.cuda.synchronize()
    assert st.item() == csa.CSA_ERR_BOUNDS
    got = cache.cpu().numpy()
    written = (got != 0).any(1).sum()
    assert written == 2   # request 0's two blocks only


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "fp4"])
@pytest.mark.parametrize("dim", [64, 128])
def test_c4_compress_index(fmt, dim):
    csa = _csa()
    x, gate, bias, cu, start, pt, n_slots, new = _compress_setup(dim, 4 + dim)
    cb = {"bf16": 2 * dim, "fp8": dim, "fp4": dim // 2}[fmt]
    codes = torch.zeros((n_slots, cb), dtype=torch.uint8, device="cuda")
    bsc = torch.zeros((n_slots, dim // 16), dtype=torch.uint8, device="cuda") if fmt == "fp4" else None
    sc = torch.zeros(n_slots, dtype=torch.float32, device="cuda") if fmt != "bf16" else None
    kind = {"bf16": csa.CSA_OUT_INDEX_BF16, "fp8": csa.CSA_OUT_INDEX_FP8,
            "fp4": csa.CSA_OUT_INDEX_FP4}[fmt]
    st = zstatus()
    csa.csa_c4_compress(dev(x), dev(gate), dev(bias), dev(cu), dev(start.astype(np.int32)),
                        int(new.max()), dev(pt), kind, codes, bsc, sc, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ys, slots = [], []
    for b in range(len(new)):
        y = orc.c4_compress(x[cu[b]:cu[b + 1]].astype(np.float64),
                            gate[cu[b]:cu[b + 1]].astype(np.float64), bias.astype(np.float64))
        for i in range(y.shape[0]):
            j = start[b] // 4 + i
            slots.append(pt[b, j // 64] * 64 + j % 64)
        ys.append(y)
    y = np.concatenate(ys)
    slots = np.asarray(slots)
    ref = orc.index_quantise(y, fmt)
    gc = codes.cpu().numpy()[slots]
    gb = bsc.cpu().numpy()[slots] if bsc is not None else None
    gs = sc.cpu().numpy()[slots] if sc is not None else None
    _compare_codes(gc, gb, gs, ref, fmt, dim, y.shape[0])


@pytest.mark.parametrize("dim", [64, 128])
def test_c4_compress_index_fp4_page(dim):
    """The compressor writing index keys into paged FP4 records gives the same
    bytes per slot as the compressor writing the plain FP4 arrays."""
    from gpu_util import fp4_page_unpack
    csa = _csa()
    x, gate, bias, cu, start, pt, n_slots, new = _compress_setup(dim, 40 + dim)
    codes = torch.zeros((n_slots, dim // 2), dtype=torch.uint8, device="cuda")
    bsc = torch.zeros((n_slots, dim // 16), dtype=torch.uint8, device="cuda")
    sc = torch.zeros(n_slots, dtype=torch.float32, device="cuda")
    rec = torch.zeros((n_slots // 64, csa.index_record_bytes(dim)), dtype=torch.uint8,
                      device="cuda")
    st = zstatus()
    args = (dev(x), dev(gate), dev(bias), dev(cu), dev(start.astype(np.int32)), int(new.max()),
            dev(pt))
    csa.csa_c4_compress(*args, csa.CSA_OUT_INDEX_FP4, codes, bsc, sc, status=st)
    csa.csa_c4_compress(*args, csa.CSA_OUT_INDEX_FP4_PAGE, rec, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    pk, pb, ps = fp4_page_unpack(rec.cpu().numpy(), dim)
    assert np.array_equal(pk, codes.cpu().numpy())
    assert np.array_equal(pb, bsc.cpu().numpy())
    assert np.array_equal(ps.view(np.uint32), sc.cpu().numpy().view(np.uint32))
    assert (ps != 0).sum() > 0


# ------------------------------------------------------------------ indexer

def _indexer_case(fmt, dim, heads, seed, c4_lens, q_lens, dist="normal"):
    rng = np.random.default_rng(seed)
    bs = len(c4_lens)
    L = np.array([4 * n + (b % 4) for b, n in enumerate(c4_lens)], dtype=np.int64)
    q_lens = np.minimum(np.asarray(q_lens), np.maximum(L, 1))
    L = np.maximum(L, q_lens)
    c4 = L // 4
    pages = np.maximum((c4 + 63) // 64, 1)
    stride = int(pages.max())
    n_pages = int(pages.sum()) + 2
    perm = rng.permutation(n_pages).astype(np.int32)
    pt = np.full((bs, stride), -1, dtype=np.int32)
    o = 0
    for b in range(bs):
        pt[b, :pages[b]] = perm[o:o + pages[b]]
        o += pages[b]
    n_slots = n_pages * 64
    key_rows, slots = [], []
    for b in range(bs):
        kr = rng.standard_t(3, (c4[b], dim)) if dist == "t3" else rng.standard_normal((c4[b], dim))
        key_rows.append(kr)
        s = np.arange(c4[b])
        slots.append(pt[b, s // 64].astype(np.int64) * 64 + s % 64)
    keys = np.concatenate(key_rows) if key_rows else np.zeros((0, dim))
    slots = np.concatenate(slots).astype(np.int64)
    ofmt = "fp4" if fmt == "fp4p" else fmt      # paged records hold the FP4 values
    kq = orc.index_quantise(keys, ofmt)
    nq = int(q_lens.sum())
    qx = rng.standard_normal((nq, heads, dim))
    qq = orc.index_quantise(qx, ofmt)
    w = rng.uniform(size=(nq, heads)).astype(np.float32)
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q_pos = np.concatenate([np.arange(L[b] - q_lens[b], L[b]) for b in range(bs)]).astype(np.int32)
    return dict(pt=pt, n_slots=n_slots, keys=kq, slots=slots, qq=qq, w=w, cu_q=cu_q, q_pos=q_pos,
                c4=c4, L=L, nq=nq, key_rows=key_rows)


INDEXER_CASES = [("bf16", 64, 8), ("fp8", 128, 64), ("fp4", 64, 8), ("fp4", 128, 64),
                 ("fp8", 64, 16), ("bf16", 128, 32), ("fp8", 128, 8), ("fp4p", 64, 8),
                 ("fp4p", 128, 64), ("fp4p", 64, 16)]


@pytest.mark.parametrize("fmt,dim,heads", INDEXER_CASES)
def test_indexer_logits(fmt, dim, heads):
    csa = _csa()
    c = _indexer_case(fmt, dim, heads, seed=dim + heads, c4_lens=[0, 1, 63, 64, 65, 1000, 5000, 2049],
                      q_lens=[1, 1, 5, 1, 2, 1, 5, 3],
                      dist="t3" if fmt in ("fp4", "fp4p") else "normal")
    kc, kb, ks = index_arrays(c["keys"], fmt, dim, c["n_slots"], c["slots"])
    qc, qb, qs = index_arrays(c["qq"], "fp4" if fmt == "fp4p" else fmt, dim, c["nq"] * heads)
    wf = c["w"] * (c["qq"]["scales"].reshape(c["nq"], heads) if fmt != "bf16" else 1.0)
    wf = wf.astype(np.float32)
    max_c4 = int(c["c4"].max())
    stride = max_c4 + 16
    logits = torch.full((c["nq"], stride), float("nan"), dtype=torch.float32, device="cuda")
    st = zstatus()
    csa.csa_indexer_logits(qc, qb, dev(wf), heads, dim, FMT[fmt], kc, kb, ks, dev(c["pt"]),
                           dev(c["c4"].astype(np.int32)), dev(c["cu_q"]), dev(c["q_pos"]), max_c4,
                           logits, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = logits.cpu().numpy()
    qd = c["qq"]["deq"].reshape(c["nq"], heads, dim)
    kd = c["keys"]["deq"]
    off = np.concatenate([[0], np.cumsum(c["c4"])])
    for b in range(len(c["c4"])):
        for t in range(c["cu_q"][b], c["cu_q"][b + 1]):
            nv = min(int(c["c4"][b]), (int(c["q_pos"][t]) + 1) // 4)
            if nv:
                ref = orc.indexer_logits(qd[t:t + 1], c["w"][t:t + 1], kd[off[b]:off[b] + c["c4"][b]],
                                         [nv])[0, :nv]
                assert rel_close(got[t, :nv], ref, 1e-2).all(), (b, t)
            assert np.isnan(got[t, nv:]).all()


@pytest.mark.parametrize("fmt,dim,heads", [("fp8", 128, 64), ("fp4", 64, 8), ("bf16", 64, 8)])
def test_indexer_logits_cuda_core_path(fmt, dim, heads):
    """Index caches whose slot count is not a multiple of 64 (here 64k + 8)
    take the CUDA-core indexer (the tensor-core kernel moves whole 64-row
    pages); same logits as the oracle to 1e-2."""
    csa = _csa()
    c = _indexer_case(fmt, dim, heads, seed=7 + dim, c4_lens=[0, 63, 65, 1000, 3000],
                      q_lens=[1, 2, 1, 5, 1], dist="t3" if fmt == "fp4" else "normal")
    n_rows = c["n_slots"] + 8
    kc, kb, ks = index_arrays(c["keys"], fmt, dim, n_rows, c["slots"])
    qc, qb, qs = index_arrays(c["qq"], fmt, dim, c["nq"] * heads)
    wf = (c["w"] * (c["qq"]["scales"].reshape(c["nq"], heads) if fmt != "bf16" else 1.0)
          ).astype(np.float32)
    max_c4 = int(c["c4"].max())
    logits = torch.full((c["nq"], max_c4 + 16), float("nan"), dtype=torch.float32, device="cuda")
    st = zstatus()
    csa.csa_indexer_logits(qc, qb, dev(wf), heads, dim, FMT[fmt], kc, kb, ks, dev(c["pt"]),
                           dev(c["c4"].astype(np.int32)), dev(c["cu_q"]), dev(c["q_pos"]), max_c4,
                           logits, num_slots=n_rows, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = logits.cpu().numpy()
    qd = c["qq"]["deq"].reshape(c["nq"], heads, dim)
    kd = c["keys"]["deq"]
    off = np.concatenate([[0], np.cumsum(c["c4"])])
    for b in range(len(c["c4"])):
        for t in range(c["cu_q"][b], c["cu_q"][b + 1]):
            nv = min(int(c["c4"][b]), (int(c["q_pos"][t]) + 1) // 4)
            if nv:
                ref = orc.indexer_logits(qd[t:t + 1], c["w"][t:t + 1],
                                         kd[off[b]:off[b] + c["c4"][b]], [nv])[0, :nv]
                assert rel_close(got[t, :nv], ref, 1e-2).all(), (b, t)
            assert np.isnan(got[t, nv:]).all()


# ------------------------------------------------------------------ top-512

def _topk_case(case, rng):
    if case == "short":
        c4, ql = [0, 1, 511, 512, 7], [1, 1, 1, 1, 1]
    elif case == "ties":
        c4, ql = [513, 2000, 8192, 8193, 20000], [1, 1, 1, 1, 1]
    elif case == "long":
        c4, ql = [262144, 100000], [1, 1]
    elif case == "causal":
        c4, ql = [3000, 9000, 700], [5, 5, 4]
    elif case == "regmax":
        # the longest rows the one-launch top-k holds in registers (32768 keys)
        c4, ql = [32768, 5, 600, 2047], [1, 1, 2, 1]
    elif case == "regmax1":
        c4, ql = [32769, 31000], [1, 1]
    elif case == "allequal_reg":
        c4, ql = [32768, 9000], [1, 1]
    elif case == "cluster2":
        # 40 rows: two CTAs per row (the four-CTA form takes up to 37 rows)
        c4, ql = [32768, 20000, 8193, 12000, 30001], [8, 8, 8, 8, 8]
    elif case == "cluster_edge":
        # rows that end just inside the second, third and fourth CTA's keys
        c4, ql = [8197, 16385, 24577, 9000, 32767], [1, 1, 1, 1, 1]
    elif case == "reg_many":
        # 80 rows: one CTA per row
        c4, ql = [32768, 9000, 20000, 1200], [20, 20, 20, 20]
    elif case == "rowmax":
        # the longest rows the one-launch top-k stages whole (49152 keys), with ties
        c4, ql = [49152, 30000, 4], [1, 3, 1]
    elif case == "rowmax1":
        # one key more: the two-stage path
        c4, ql = [49153, 2], [1, 1]
    else:
        c4, ql = [50000, 1000], [1, 1]
    c4 = np.asarray(c4, dtype=np.int64)
    ql = np.asarray(ql)
    L = 4 * c4 + 3
    bs = len(c4)
    pages = np.maximum((c4 + 63) // 64, 1)
    stride = int(pages.max())
    n_pages = int(pages.sum()) + 5
    perm = rng.permutation(n_pages).astype(np.int32)
    pt = np.full((bs, stride), -1, dtype=np.int32)
    o = 0
    for b in range(bs):
        pt[b, :pages[b]] = perm[o:o + pages[b]]
        o += pages[b]
    nq = int(ql.sum())
    cu_q = np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)
    q_pos = np.concatenate([np.arange(L[b] - ql[b], L[b]) for b in range(bs)]).astype(np.int32)
    max_c4 = int(c4.max())
    stride_l = max_c4 + 3
    lg = np.full((nq, stride_l), np.nan, dtype=np.float32)
    for t in range(nq):
        if case in ("ties", "rowmax", "rowmax1", "regmax", "regmax1", "cluster2"):
            v = np.round(rng.standard_normal(max_c4) * 3) / 2
            v[rng.integers(0, max_c4, 50)] = -0.0
        elif case in ("allequal", "allequal_reg"):
            v = np.full(max_c4, 2.5)
        elif case == "cluster_edge":
            v = np.maximum(rng.standard_normal(max_c4), 0.0) * 3
        elif case == "long":
            v = rng.standard_t(3, max_c4)
            v[rng.integers(0, max_c4, 100)] = -np.inf
        else:
            v = rng.standard_normal(max_c4)
        lg[t, :max_c4] = v.astype(np.float32)
    # entries beyond each row's visible length must be ignored
    b_of = np.repeat(np.arange(bs), ql)
    nv = np.array([min(int(c4[b_of[t]]), (int(q_pos[t]) + 1) // 4) for t in range(nq)])
    for t in range(nq):
        lg[t, nv[t]:] = np.nan
    return dict(c4=c4, pt=pt, n_slots=n_pages * 64, cu_q=cu_q, q_pos=q_pos, lg=lg, nv=nv, b_of=b_of,
                max_c4=max_c4, nq=nq)


@pytest.mark.parametrize("case", ["short", "ties", "long", "causal", "allequal", "rowmax",
                                  "rowmax1", "regmax", "regmax1", "allequal_reg", "cluster2",
                                  "cluster_edge", "reg_many"])
def test_topk512_bit_exact(case):
    csa = _csa()
    c = _topk_case(case, np.random.default_rng(len(case)))
    out = torch.full((c["nq"], 512), -7, dtype=torch.int32, device="cuda")
    raw = torch.full((c["nq"], 512), -7, dtype=torch.int32, device="cuda")
    st = zstatus()
    csa.csa_topk512_page_transform(dev(c["lg"]), dev(c["c4"].astype(np.int32)), dev(c["cu_q"]),
                                   dev(c["q_pos"]), dev(c["pt"]), c["n_slots"], c["max_c4"], out, raw,
                                   status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    go, gr = out.cpu().numpy(), raw.cpu().numpy()
    for t in range(c["nq"]):
        phys, logical = orc.topk_transform(c["lg"][t], int(c["nv"][t]), c["pt"][c["b_of"][t]],
                                           c["n_slots"])
        assert np.array_equal(gr[t], logical), t
        assert np.array_equal(go[t], phys), t


def test_topk512_nan_reported_and_ranked_last():
    csa = _csa()
    rng = np.random.default_rng(5)
    n = 3000
    lg = rng.standard_normal((1, n)).astype(np.float32)
    lg[0, [7, 100, 2999]] = np.nan
    pt = np.arange(47, dtype=np.int32)[None]
    out = torch.empty((1, 512), dtype=torch.int32, device="cuda")
    raw = torch.empty((1, 512), dtype=torch.int32, device="cuda")
    st = zstatus()
    csa.csa_topk512_page_transform(dev(lg), dev(np.array([n], np.int32)), dev(np.array([0, 1], np.int32)),
                                   None, dev(pt), 47 * 64, n, out, raw, status=st)
    torch.cuda.synchronize()
    assert st.item() == csa.CSA_ERR_NAN
    clean = lg.copy()
    clean[np.isnan(clean)] = -np.inf
    phys, logical = orc.topk_transform(clean[0], n, pt[0], 47 * 64)
    assert np.array_equal(raw.cpu().numpy()[0], logical)


def test_topk512_bad_page_reported():
    csa = _csa()
    lg = np.arange(200, dtype=np.float32)[None]
    pt = np.array([[0, 9]], dtype=np.int32)       # page 9 is beyond a 2-page pool
    out = torch.empty((1, 512), dtype=torch.int32, device="cuda")
    st = zstatus()
    csa.csa_topk512_page_transform(dev(lg), dev(np.array([100], np.int32)),
                                   dev(np.array([0, 1], np.int32)), None, dev(pt), 128, 200, out,
                                   status=st)
    torch.cuda.synchronize()
    assert st.item() == csa.CSA_ERR_BOUNDS
    o = out.cpu().numpy()[0]
    assert np.array_equal(o[:64], np.arange(64)) and (o[64:100] == -1).all() and (o[100:] == -1).all()


# ------------------------------------------------------------------ attention

def _attn_case(kv_fmt, heads, decode, seed, L=(300, 5000, 70000), q_lens=(7, 1, 20), window=128):
    rng = np.random.default_rng(seed)
    L = np.asarray(L, dtype=np.int64)
    bs = len(L)
    q_lens = np.ones(bs, dtype=np.int64) if decode else np.asarray(q_lens)
    c4 = L // 4
    pages = (L + 255) // 256
    stride = int(pages.max())
    n_pages = int(pages.sum()) + 2
    perm = rng.permutation(n_pages).astype(np.int32)
    pt = np.full((bs, stride), -1, dtype=np.int32)
    o = 0
    for b in range(bs):
        pt[b, :pages[b]] = perm[o:o + pages[b]]
        o += pages[b]
    fp8 = kv_fmt == "fp8"
    rb = 656 if fp8 else 1152
    c4_cache = np.zeros((n_pages * 64, rb), dtype=np.uint8)
    raw_cache = np.zeros((n_pages * 256, rb), dtype=np.uint8)
    nq = int(q_lens.sum())
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q_pos = np.concatenate([np.arange(L[b] - q_lens[b], L[b]) for b in range(bs)]).astype(np.int32)
    idx = np.full((nq, 512), -1, dtype=np.int32)
    c4_rows, raw_rows = {}, {}
    for b in range(bs):
        rows = rng.standard_normal((c4[b], 576)) * (1 + 2 * (b == 1))
        enc = orc.kv_encode_rows(rows, fp8)
        s = np.arange(c4[b])
        sl = pt[b, s // 64].astype(np.int64) * 64 + s % 64
        c4_cache[sl] = enc
        c4_rows[b] = orc.kv_decode_rows(enc, fp8)
        lo = max(0, int(L[b] - q_lens[b]) - window + 1)
        pos = np.arange(lo, L[b])
        rr = rng.standard_normal((len(pos), 576))
        renc = orc.kv_encode_rows(rr, fp8)
        rsl = pt[b, pos // 256].astype(np.int64) * 256 + pos % 256
        raw_cache[rsl] = renc
        raw_rows[b] = dict(zip(pos.tolist(), orc.kv_decode_rows(renc, fp8)))
    chosen = {}
    for t in range(nq):
        b = int(np.searchsorted(cu_q, t, side="right") - 1)
        nv = min(int(c4[b]), (int(q_pos[t]) + 1) // 4)
        if nv <= 512:
            sel = np.arange(nv)
        else:
            sel = np.sort(rng.choice(nv, 512, replace=False))
        lst = np.full(512, -1, dtype=np.int64)
        lst[:len(sel)] = sel
        if t == 1 and len(sel) > 40:          # holes in the middle are allowed
            lst[10:20] = -1
        chosen[t] = lst[lst >= 0]
        ok = lst >= 0
        idx[t, ok] = pt[b, lst[ok] // 64] * 64 + lst[ok] % 64
    q = torch.randn((nq, heads, 576), generator=torch.Generator().manual_seed(seed)).bfloat16()
    return dict(pt=pt, c4_cache=c4_cache, raw_cache=raw_cache, idx=idx, q=q, cu_q=cu_q, q_pos=q_pos,
                L=L, c4_rows=c4_rows, raw_rows=raw_rows, chosen=chosen, nq=nq, window=window)


@pytest.mark.parametrize("kv_fmt,heads,decode", [("fp8", 64, True), ("bf16", 16, True),
                                                 ("fp8", 64, False), ("bf16", 32, False),
                                                 ("fp8", 128, True), ("bf16", 64, True)])
def test_sparse_mqa(kv_fmt, heads, decode):
    csa = _csa()
    c = _attn_case(kv_fmt, heads, decode, seed=heads + decode)
    sm_scale = 1.0 / math.sqrt(576) * (3.0 if heads == 128 else 1.0)
    out = torch.empty((c["nq"], heads, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((c["nq"], heads), dtype=torch.float32, device="cuda")
    st = zstatus()
    fn = csa.csa_sparse_mqa_decode if decode else csa.csa_sparse_mqa_prefill
    fn(c["q"].cuda(), dev(c["c4_cache"]), dev(c["raw_cache"]), FMT[kv_fmt], dev(c["idx"]),
       dev(c["pt"]), dev(c["L"].astype(np.int32)), dev(c["cu_q"]), dev(c["q_pos"]), c["window"],
       sm_scale, out, lse, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    go = out.float().cpu().numpy()
    gl = lse.cpu().numpy()
    tol = 2e-2 if kv_fmt == "fp8" else 5e-3
    qf = c["q"].double().numpy()
    for t in range(c["nq"]):
        b = int(np.searchsorted(c["cu_q"], t, side="right") - 1)
        win = orc.window_positions(int(c["q_pos"][t]), c["window"])
        rows = np.concatenate([c["c4_rows"][b][c["chosen"][t]].reshape(-1, 576),
                               np.array([c["raw_rows"][b][int(r)] for r in win]).reshape(-1, 576)])
        ro, rl = orc.sparse_attention(qf[t], rows, sm_scale)
        # outputs are bf16: the bound is the tolerance plus half a bf16 ulp of
        # the reference (only matters for |out| > 1, as in the x3 request)
        err = np.abs(go[t] - ro) - bf16_bound(ro, rel=0.0)
        assert err.max() <= tol, (t, err.max())
        assert np.abs(gl[t] - rl).max() <= 2e-2, t


def test_sparse_mqa_window_only_and_zero_window():
    """No selected rows: the window alone; window 0 with rows: compressed only."""
    csa = _csa()
    c = _attn_case("bf16", 16, True, seed=9, L=(900, 3000))
    idx = np.full_like(c["idx"], -1)
    out = torch.empty((c["nq"], 16, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((c["nq"], 16), dtype=torch.float32, device="cuda")
    csa.csa_sparse_mqa_decode(c["q"].cuda(), dev(c["c4_cache"]), dev(c["raw_cache"]), 0, dev(idx),
                              dev(c["pt"]), dev(c["L"].astype(np.int32)), dev(c["cu_q"]), None, 128,
                              0.05, out, lse)
    torch.cuda.synchronize()
    go = out.float().cpu().numpy()
    qf = c["q"].double().numpy()
    for t in range(c["nq"]):
        win = orc.window_positions(int(c["q_pos"][t]), 128)
        rows = np.array([c["raw_rows"][t][int(r)] for r in win])
        ro, _ = orc.sparse_attention(qf[t], rows, 0.05)
        assert (np.abs(go[t] - ro) - bf16_bound(ro, rel=0.0)).max() <= 5e-3
    csa.csa_sparse_mqa_decode(c["q"].cuda(), dev(c["c4_cache"]), dev(c["raw_cache"]), 0,
                              dev(c["idx"]), dev(c["pt"]), dev(c["L"].astype(np.int32)),
                              dev(c["cu_q"]), None, 0, 0.05, out, lse)
    torch.cuda.synchronize()
    go = out.float().cpu().numpy()
    for t in range(c["nq"]):
        rows = c["c4_rows"][t][c["chosen"][t]]
        ro, _ = orc.sparse_attention(qf[t], rows, 0.05)
        assert (np.abs(go[t] - ro) - bf16_bound(ro, rel=0.0)).max() <= 5e-3
