"""Failure detection without a GPU fault: a bounded device wait that nothing
completes gives up after the library's limit, records CSA_ERR_TIMEOUT in the
caller's status word, and the context keeps working; bad pages and lengths
are reported as CSA_ERR_BOUNDS (see test_gpu_steps for those cases)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    from compressed_sparse_attention_12_b200 import build, csa
    build.build()
    return csa.lib()


def test_bounded_wait_times_out_and_the_context_stays_usable():
    from compressed_sparse_attention_12_b200 import csa
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa.csa_selftest_wait_timeout(st, waited)
    torch.cuda.synchronize()
    assert st.item() == csa.CSA_ERR_TIMEOUT
    assert 0.9e9 <= waited.item() <= 1.5e9
    # an earlier code is kept
    st.fill_(csa.CSA_ERR_BOUNDS)
    csa.csa_selftest_wait_timeout(st)
    torch.cuda.synchronize()
    assert st.item() == csa.CSA_ERR_BOUNDS
    # the context still runs work: store and read back one KV row
    rows = torch.randn(3, 576, device="cuda")
    cache = torch.zeros((8, 1152), dtype=torch.uint8, device="cuda")
    st.zero_()
    csa.csa_kv_store(rows, torch.tensor([5, 0, 2], dtype=torch.int32, device="cuda"),
                     csa.CSA_FMT_BF16, cache, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = cache[5].cpu().numpy().view(np.uint16)[:576]
    want = rows[0].bfloat16().cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
