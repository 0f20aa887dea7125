"""Host logic of the synthetic workloads: page tables are permutations of the
page pool, the HCA plan hands the compressor exactly the blocks completed by
the step's query tokens, and the DSA table covers every raw token."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
from compressed_sparse_attention_12_b200 import synth  # noqa: E402


@pytest.mark.parametrize("name,scale", [("decode_128k", 1 / 64), ("ragged", 1 / 64),
                                        ("prefill", 1 / 16)])
def test_page_table_is_a_permutation(name, scale):
    w = synth.workload(name, scale)
    pt = synth.page_table(w)
    used = pt[pt >= 0]
    assert len(np.unique(used)) == used.size
    assert used.max() < w.num_pages
    for b, n in enumerate(w.pages_per_req):
        assert (pt[b, :n] >= 0).all() and (pt[b, n:] == -1).all()


def test_dsa_page_table_covers_every_token_once():
    w = synth.workload("dsa_128k", 1 / 64)
    pt = synth.dsa_page_table(w)
    per = (w.seq_lens + 63) // 64
    used = pt[pt >= 0]
    assert len(np.unique(used)) == used.size == per.sum()
    assert (pt[:, :per.max()] >= 0).all()


@pytest.mark.parametrize("L,Q", [(131072, 1), (131071, 1), (300, 40), (128 * 40 + 7, 1),
                                 (100, 1), (4160, 64), (16640, 256)])
def test_hca_plan_pools_the_blocks_completed_by_this_step(L, Q):
    w = synth.Workload("t", [L], [Q], 8, 64, "bf16", 16, "bf16", new_tokens=[0])
    start, new, direct = synth.hca_plan(w)
    # blocks j with 128j+127 among the query positions L-Q .. L-1
    want = [j for j in range(L // 128) if L - Q <= 128 * j + 127 <= L - 1]
    if want:
        assert start[0] == 128 * want[0] and new[0] == L - start[0]
        assert new[0] // 128 == len(want)
        assert direct[0] == want[0]
    else:
        assert new[0] == 0 and direct[0] == L // 128
    assert start[0] % 128 == 0 or new[0] == 0


def test_hca_draw_shapes():
    w = synth.workload("hca_prefill", 1 / 16)
    d = synth.draw_hca(w, "cpu")
    start, new, direct = synth.hca_plan(w)
    assert d["hca_kv"].shape == (int(direct.sum()), 576)
    assert d["raw_kv"].shape == (int(new.sum()), 576)
    assert d["bias"].shape == (128, 576)
    # the compressor's rows are the raw rows at [start, L)
    sel = (d["raw_req"] == 0) & (d["raw_pos"] >= start[0])
    assert np.array_equal(d["kv_raw"][np.nonzero(sel)[0]].numpy(), d["raw_kv"].numpy())
