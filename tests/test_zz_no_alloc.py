"""GPU test of csa_topk512_page_transform_noalloc, the top-512 entry point for
callers that cannot pass a workspace or allocate device memory when they call
(plugin interfaces that hand over only inputs and outputs; hot paths that must
not reach the allocator).  Its scratch is a fixed device array inside the
library; its results must equal those of csa_topk512_page_transform, which
takes a caller workspace, bit for bit, on consecutive calls (the array keeps
the previous call's contents).  Collected last so that a run stopping at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _case(rng, c4_lens, q_lens):
    c4 = np.asarray(c4_lens, dtype=np.int64)
    ql = np.asarray(q_lens, dtype=np.int64)
    L = 4 * c4 + 3
    bs = len(c4)
    pages = np.maximum((c4 + 63) // 64, 1)
    n_pages = int(pages.sum()) + 3
    perm = rng.permutation(n_pages).astype(np.int32)
    pt = np.full((bs, int(pages.max())), -1, dtype=np.int32)
    o = 0
    for b in range(bs):
        pt[b, :pages[b]] = perm[o:o + pages[b]]
        o += pages[b]
    nq = int(ql.sum())
    cu_q = np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)
    q_pos = np.concatenate([np.arange(L[b] - ql[b], L[b]) for b in range(bs)]).astype(np.int32)
    max_c4 = int(c4.max())
    lg = (np.round(rng.standard_normal((nq, max_c4 + 5)) * 8) / 4).astype(np.float32)  # ties
    lg[:, ::97] = -0.0
    d = lambda a: torch.as_tensor(np.ascontiguousarray(a), device="cuda")
    return dict(lg=d(lg), c4=d(c4.astype(np.int32)), cu_q=d(cu_q), q_pos=d(q_pos), pt=d(pt),
                n_slots=n_pages * 64, max_c4=max_c4, nq=nq)


def test_noalloc_equals_workspace_entry_point_on_consecutive_calls():
    from compressed_sparse_attention_12_b200 import build, csa
    build.build()
    rng = np.random.default_rng(2024)
    cases = [_case(rng, [300, 9000, 70000], [1, 3, 2]),
             _case(rng, [262144, 511, 40000, 7], [1, 1, 4, 1]),
             # 4100 rows of short lists: one launch with no scratch, accepted
             # although a two-stage workspace for them would exceed the array
             _case(rng, [1000] * 41, [100] * 41)]
    assert csa.csa_topk512_workspace_size(41 * 100, 1000) > csa.TOPK_NOALLOC_MAX_BYTES
    for c in cases:                     # two calls in a row, different sizes
        st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
        st_na = torch.zeros(1, dtype=torch.int32, device="cuda")
        ref = torch.full((c["nq"], 512), -7, dtype=torch.int32, device="cuda")
        ref_raw = torch.full_like(ref, -7)
        got = torch.full_like(ref, -9)
        got_raw = torch.full_like(ref, -9)
        csa.csa_topk512_page_transform(c["lg"], c["c4"], c["cu_q"], c["q_pos"], c["pt"],
                                       c["n_slots"], c["max_c4"], ref, ref_raw, status=st_ref)
        csa.csa_topk512_page_transform_noalloc(c["lg"], c["c4"], c["cu_q"], c["q_pos"], c["pt"],
                                               c["n_slots"], c["max_c4"], got, got_raw,
                                               status=st_na)
        torch.cuda.synchronize()
        assert st_ref.item() == 0 and st_na.item() == 0
        assert torch.equal(got, ref)
        assert torch.equal(got_raw, ref_raw)
        assert (got_raw >= 0).sum().item() > 0


def test_noalloc_rejects_sizes_beyond_its_array():
    from compressed_sparse_attention_12_b200 import build, csa
    build.build()
    L = csa.lib()
    p = lambda: ctypes.c_void_p(4096)        # never dereferenced: rejected on the host
    # rows longer than 49152 keys take the two-stage selection, whose
    # candidates (512 rows x 8 chunks x (512 x 8 + 8) B) exceed 16 MiB
    num_q, max_c4 = 512, 65536
    assert csa.csa_topk512_workspace_size(num_q, max_c4) > csa.TOPK_NOALLOC_MAX_BYTES
    r = L.csa_topk512_page_transform_noalloc(p(), max_c4, num_q, p(), 1, p(), None, p(), 128,
                                             128 * 64, 64, max_c4, p(), None, None, None)
    assert r == csa.CSA_ERR_WORKSPACE
