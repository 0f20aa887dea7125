"""The DSA comparison path and the fused rotary embedding on the GPU against
the oracle ("Token 的一生：DSV4 架构与 DSpark" §1 从 DSA 到 DSV4, §3.1, §4):
plain (unrotated) quantisation, RoPE -> Hadamard -> quant for index queries
and keys (also inside the compressor), and the whole DSA step (store, indexer
over raw tokens with keys s <= p, top-512 with 64-token pages, attention over
the selected raw rows) at oracle-sized and full benchmark sizes."""
import math

import numpy as np
import pytest
import torch

from gpu_util import bf16_bound, dev, rel_close
from oracle import oracle as orc
from test_gpu_steps import _compare_codes, _compress_setup

pytestmark = pytest.mark.gpu
FMT = {"bf16": 0, "fp8": 1, "fp4": 2}


@pytest.fixture(scope="module", autouse=True)
def lib():
    from compressed_sparse_attention_12_b200 import build, csa
    build.build()
    return csa.lib()


def _csa():
    from compressed_sparse_attention_12_b200 import csa
    return csa


def _zst():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _outs(fmt, dim, rows, fill=None):
    cb = {"bf16": 2 * dim, "fp8": dim, "fp4": dim // 2}[fmt]
    mk = (lambda shape, dt: torch.full(shape, fill, dtype=dt, device="cuda")) if fill is not None \
        else (lambda shape, dt: torch.zeros(shape, dtype=dt, device="cuda"))
    codes = mk((rows, cb), torch.uint8)
    bsc = mk((rows, dim // 16), torch.uint8) if fmt == "fp4" else None
    sc = mk((rows,), torch.float32) if fmt != "bf16" else None
    return codes, bsc, sc


def _host(t):
    return None if t is None else t.cpu().numpy()


@pytest.mark.parametrize("fmt", ["fp8", "fp4", "bf16"])
@pytest.mark.parametrize("dim", [64, 128])
def test_index_quant_without_rotation(fmt, dim):
    csa = _csa()
    g = torch.Generator().manual_seed(dim + len(fmt))
    rows = 2000
    x = torch.randn(rows, dim, generator=g)
    x[::5] *= 30.0
    x[1] = 0.0
    w = torch.rand(rows, generator=g)
    codes, bsc, sc = _outs(fmt, dim, rows)
    wo = torch.empty(rows, dtype=torch.float32, device="cuda")
    st = _zst()
    csa.csa_index_quant(x.cuda(), FMT[fmt], codes, bsc, sc, w_in=w.cuda(), w_out=wo, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = orc.dsa_index_quantise(x.double().numpy(), fmt)
    _compare_codes(_host(codes), _host(bsc), _host(sc), ref, fmt, dim, rows)
    want = w.numpy() * (_host(sc) if sc is not None else 1.0)
    assert np.array_equal(wo.cpu().numpy(), want.astype(np.float32))


@pytest.mark.parametrize("fmt", ["fp8", "fp4", "bf16"])
@pytest.mark.parametrize("dim,rope_dim,heads", [(128, 64, 8), (64, 64, 4), (128, 128, 1),
                                                (64, 16, 2)])
def test_rope_hadamard_quant(fmt, dim, rope_dim, heads):
    from compressed_sparse_attention_12_b200 import synth
    csa = _csa()
    g = torch.Generator().manual_seed(dim * 3 + rope_dim + heads + len(fmt))
    n_tok, max_pos = 700, 1 << 17
    x = torch.randn(n_tok, heads, dim, generator=g).bfloat16()
    pos = torch.randint(0, max_pos, (n_tok,), generator=g, dtype=torch.int32)
    pos[0], pos[1] = 0, max_pos - 1
    freqs = synth.rope_freqs(max_pos, rope_dim)
    w = torch.rand(n_tok, heads, generator=g)
    codes, bsc, sc = _outs(fmt, dim, n_tok * heads)
    wo = torch.empty(n_tok, heads, dtype=torch.float32, device="cuda")
    st = _zst()
    csa.csa_rope_hadamard_quant(x.cuda(), freqs.cuda(), rope_dim, pos.cuda(), heads, FMT[fmt],
                                codes, bsc, sc, w_in=w.cuda(), w_out=wo, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = orc.rope_index_quantise(x.double().numpy(), freqs.numpy(), rope_dim,
                                  pos.numpy()[:, None], fmt)
    _compare_codes(_host(codes), _host(bsc), _host(sc), ref, fmt, dim, n_tok * heads)


def test_rope_position_out_of_range_is_reported():
    from compressed_sparse_attention_12_b200 import synth
    csa = _csa()
    x = torch.randn(4, 128).cuda()
    pos = torch.tensor([0, 5, 99, -1], dtype=torch.int32, device="cuda")
    codes, _, sc = _outs("fp8", 128, 4, fill=0x5A)
    st = _zst()
    csa.csa_rope_hadamard_quant(x, synth.rope_freqs(64, 64).cuda(), 64, pos, 1, FMT["fp8"],
                                codes, None, sc, status=st)
    torch.cuda.synchronize()
    assert st.item() == csa.CSA_ERR_BOUNDS
    got = codes.cpu().numpy()
    assert (got[2] == 0x5A).all() and (got[3] == 0x5A).all()
    assert not (got[0] == 0x5A).all()


@pytest.mark.parametrize("fmt", ["fp8", "fp4"])
@pytest.mark.parametrize("dim", [64, 128])
def test_c4_compress_index_rope(fmt, dim):
    from compressed_sparse_attention_12_b200 import synth
    csa = _csa()
    x, gate, bias, cu, start, pt, n_slots, new = _compress_setup(dim, 40 + dim)
    rope_dim = 64
    freqs = synth.rope_freqs(1 << 15, rope_dim)
    codes, bsc, sc = _outs(fmt, dim, n_slots)
    kind = {"fp8": csa.CSA_OUT_INDEX_FP8, "fp4": csa.CSA_OUT_INDEX_FP4}[fmt]
    st = _zst()
    csa.csa_c4_compress_index_rope(dev(x), dev(gate), dev(bias), dev(cu),
                                   dev(start.astype(np.int32)), int(new.max()), dev(pt), kind,
                                   freqs.cuda(), rope_dim, codes, bsc, sc, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ys, slots, kpos = [], [], []
    for b in range(len(new)):
        y = orc.c4_compress(x[cu[b]:cu[b + 1]].astype(np.float64),
                            gate[cu[b]:cu[b + 1]].astype(np.float64), bias.astype(np.float64))
        for i in range(y.shape[0]):
            j = start[b] // 4 + i
            slots.append(pt[b, j // 64] * 64 + j % 64)
            kpos.append(4 * j)
        ys.append(y)
    y = np.concatenate(ys)
    slots = np.asarray(slots)
    ref = orc.rope_index_quantise(y, freqs.numpy(), rope_dim, np.asarray(kpos), fmt)
    _compare_codes(_host(codes)[slots], None if bsc is None else _host(bsc)[slots],
                   _host(sc)[slots], ref, fmt, dim, y.shape[0])


def _dsa_check(scale, sample_req=None):
    from compressed_sparse_attention_12_b200 import pipeline, synth
    w = synth.workload("dsa_128k", scale)
    data = synth.draw_dsa(w, "cuda")
    batch = pipeline.DsaBatch(w, data)
    batch.logits.fill_(float("nan"))
    batch.step()
    torch.cuda.synchronize()
    batch.check_status()
    ref = orc.dsa_step(w, data, batch.pt_host, requests=sample_req, sm_scale=batch.sm_scale)
    raw = batch.raw_indices.cpu().numpy()
    phys = batch.indices.cpu().numpy()
    lg = batch.logits.cpu().numpy()
    out = batch.out.float().cpu().numpy()
    overlaps, exact = [], 0
    for t, r in ref.items():
        n = r["n_vis"]
        assert rel_close(lg[t, :n], r["logits"], 1e-2).all(), t
        want = set(r["logical"][r["logical"] >= 0].tolist())
        got = set(raw[t][raw[t] >= 0].tolist())
        assert len(got) == len(want) == min(512, n)
        g = raw[t][raw[t] >= 0]
        assert np.array_equal(phys[t][:len(g)], batch.pt_host[t, g // 64] * 64 + g % 64)
        overlaps.append(len(got & want) / len(want))
        if got == want:
            exact += 1
            err = np.abs(out[t] - r["out"]) - bf16_bound(r["out"], rel=0.0)
            assert err.max() <= 2e-2, (t, err.max())
            assert np.abs(batch.lse.cpu().numpy()[t] - r["lse"]).max() <= 2e-2
        # top-512 bit-exact when both sides select on the oracle's logits
        lg32 = np.zeros((1, batch.logit_stride), np.float32)
        lg32[0, :n] = r["logits"].astype(np.float32)
        csa = _csa()
        o1 = torch.empty((1, 512), dtype=torch.int32, device="cuda")
        o2 = torch.empty((1, 512), dtype=torch.int32, device="cuda")
        st = _zst()
        csa.csa_dsa_topk512_page_transform(dev(lg32), batch.seq_lens[t:t + 1],
                                           dev(np.array([0, 1], np.int32)),
                                           batch.q_pos[t:t + 1], batch.page_table[t:t + 1],
                                           batch.slots_n, n, o1, o2, status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        p_ref, l_ref = orc.topk_transform(lg32[0], n, batch.pt_host[t], batch.slots_n,
                                          c4_page_size=64)
        assert np.array_equal(o2.cpu().numpy()[0], l_ref)
        assert np.array_equal(o1.cpu().numpy()[0], p_ref)
    print(f"\ndsa scale {scale}: mean top-512 overlap {np.mean(overlaps):.5f}, "
          f"identical sets {exact}/{len(ref)}")
    assert np.mean(overlaps) >= 0.98
    assert exact >= 0.5 * len(ref)


def test_dsa_step_end_to_end():
    _dsa_check(1 / 64)


def test_dsa_full_size_sampled():
    _dsa_check(1.0, sample_req=[0, 17, 31])
