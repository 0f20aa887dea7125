"""The C ABI library loads on a machine without a GPU, exports every entry
point include/csa.h declares, and rejects malformed arguments on the host
before any launch (no GPU calls are made here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(csa_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from compressed_sparse_attention_12_b200 import build, csa
    build.build()
    return csa.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    from compressed_sparse_attention_12_b200 import csa
    assert set(names) <= set(csa.EXPORTED) | {"csa_status_string"}


def test_status_strings_and_constants(L):
    from compressed_sparse_attention_12_b200 import csa
    assert csa.status_string(0) == "ok"
    for c in range(1, 8):
        assert csa.status_string(c) not in ("ok", "unknown status")
    assert csa.status_string(99) == "unknown status"
    assert csa.csa_abi_version() == 1
    assert csa.csa_kv_row_bytes(csa.CSA_FMT_FP8) == 656
    assert csa.csa_kv_row_bytes(csa.CSA_FMT_BF16) == 1152
    assert csa.csa_kv_row_bytes(7) == 0


def test_workspace_sizes(L):
    from compressed_sparse_attention_12_b200 import csa
    assert csa.csa_topk512_workspace_size(0, 100) == 0
    # per row and 8192-logit chunk: 512 (key, index) candidate pairs and one
    # (512th key, largest key) pair
    assert csa.csa_topk512_workspace_size(3, 8192) == 3 * 1 * (512 * 8 + 8)
    assert csa.csa_topk512_workspace_size(3, 8193) == 3 * 2 * (512 * 8 + 8)
    # up to 64 rows longer than 49152 logits take the bound-first selection:
    # per row 2048 group maxima, one count per 4096-logit chunk, and two
    # (key, index) buffers as long as the row
    assert csa.csa_topk512_workspace_size(8, 262144) == (8 * 2048 * 4 + 8 * 64 * 4 +
                                                         4 * 8 * 262144 * 4)
    assert csa.csa_topk512_workspace_size(65, 262144) == 65 * 32 * (512 * 8 + 8)
    assert csa.csa_sparse_mqa_workspace_size(4096, 64, 128, 0) == 0
    assert csa.csa_sparse_mqa_workspace_size(32, 64, 128, 1) > 0


def _p(v=1):
    return ctypes.c_void_p(v * 256)   # never dereferenced: host checks fail first


def test_host_validation_rejects_before_launch(L):
    from compressed_sparse_attention_12_b200 import csa
    # page size other than 64
    r = L.csa_topk512_page_transform(_p(), 64, 1, _p(), 1, _p(), None, _p(), 4, 256, 32, 64,
                                     _p(), None, _p(), 1 << 20, None, None)
    assert r == csa.CSA_ERR_INVALID
    # workspace too small
    r = L.csa_topk512_page_transform(_p(), 64, 1, _p(), 1, _p(), None, _p(), 4, 256, 64, 64,
                                     _p(), None, _p(), 8, None, None)
    assert r == csa.CSA_ERR_WORKSPACE
    # unsupported index dim / format / heads
    r = L.csa_hadamard_quant(_p(), csa.CSA_FMT_BF16, 4, 96, csa.CSA_FMT_FP8, None, 0, _p(), None,
                             _p(), None, None, None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    r = L.csa_hadamard_quant(_p(), csa.CSA_FMT_BF16, 4, 128, 9, None, 0, _p(), None, _p(), None,
                             None, None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    # FP4 without block scales
    r = L.csa_hadamard_quant(_p(), csa.CSA_FMT_BF16, 4, 128, csa.CSA_FMT_FP4, None, 0, _p(), None,
                             _p(), None, None, None, None)
    assert r == csa.CSA_ERR_INVALID
    r = L.csa_indexer_logits(_p(), None, _p(), 1, 200, 128, csa.CSA_FMT_FP8, _p(), None, _p(), 64,
                             _p(), 1, _p(), 1, _p(), None, 64, _p(), 64, None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    # logits row stride shorter than the longest row
    r = L.csa_indexer_logits(_p(), None, _p(), 1, 64, 128, csa.CSA_FMT_FP8, _p(), None, _p(), 64,
                             _p(), 1, _p(), 1, _p(), None, 100, _p(), 64, None, None)
    assert r == csa.CSA_ERR_INVALID
    # KV compress needs dim 576; index compress needs 64/128
    r = L.csa_c4_compress(_p(), _p(), _p(), 512, 1, _p(), 8, _p(), 8, _p(), 4,
                          csa.CSA_OUT_KV_FP8, _p(), None, None, 64, None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    r = L.csa_c4_compress(_p(), _p(), _p(), 576, 1, _p(), 8, _p(), 8, _p(), 4,
                          csa.CSA_OUT_INDEX_FP8, _p(), None, None, 64, None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    # attention: heads not a multiple of 16, window out of range, bad KV format
    args = [_p(), 1, 24, _p(), _p(), csa.CSA_FMT_FP8, 64, 256, _p(), _p(), 1, _p(), 1, _p(), None,
            128, 0.1, _p(), None, _p(), 1 << 30, None, None]
    assert L.csa_sparse_mqa_decode(*args) == csa.CSA_ERR_UNSUPPORTED
    args[2] = 64
    args[15] = 5000
    assert L.csa_sparse_mqa_decode(*args) == csa.CSA_ERR_UNSUPPORTED
    args[15] = 128
    args[5] = csa.CSA_FMT_FP4
    assert L.csa_sparse_mqa_prefill(*args) == csa.CSA_ERR_UNSUPPORTED
    # q_pos NULL needs one query per request
    args[5] = csa.CSA_FMT_FP8
    args[1] = 3
    assert L.csa_sparse_mqa_prefill(*args) == csa.CSA_ERR_INVALID
    # empty work is a no-op
    assert L.csa_kv_store(None, 0, None, csa.CSA_FMT_FP8, None, 0, None, None) == csa.CSA_OK
    assert L.csa_kv_store(None, 4, None, 5, None, 0, None, None) == csa.CSA_ERR_UNSUPPORTED


def test_product_path_has_no_oracle_dependency():
    """The library package never imports or loads the oracle."""
    pkg = os.path.join(ROOT, "compressed_sparse_attention_12_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"(import|from)\s+oracle|liboracle|csa_oracle", txt), f


def test_generic_workspace_size_matches_the_per_operation_calls():
    from compressed_sparse_attention_12_b200 import csa
    assert csa.csa_workspace_size(csa.CSA_OP_TOPK512, max_rows=32, max_len=32768) == \
        csa.csa_topk512_workspace_size(32, 32768)
    assert csa.csa_workspace_size(csa.CSA_OP_INDEXER_TOPK512, bs=32, max_rows=32, max_len=32768,
                                  heads=64, idx_dim=128, fmt=csa.CSA_FMT_FP8) == \
        csa.csa_indexer_topk512_workspace_size(32, 32, 64, 128, csa.CSA_FMT_FP8, 32768)
    assert csa.csa_workspace_size(csa.CSA_OP_SPARSE_MQA, max_rows=32, heads=64, window=128,
                                  decode=True) == csa.csa_sparse_mqa_workspace_size(32, 64, 128, True)
    assert csa.csa_workspace_size(csa.CSA_OP_HCA_ATTENTION, max_rows=32, heads=64, window=128,
                                  decode=True, max_len=1024) == \
        csa.csa_hca_attention_workspace_size(32, 64, 128, True, 1024)
    assert csa.csa_workspace_size(99) == 0


def test_host_validation_of_the_next_rows(L):
    """HCA, fused RoPE, DSA, unrotated quantisation and the wait self-test
    reject bad arguments on the host, before any launch."""
    from compressed_sparse_attention_12_b200 import csa
    # HCA compressor: KV output kinds only, dim 576
    r = L.csa_hca_compress(_p(), _p(), _p(), 576, 1, _p(), 256, _p(), 256, _p(), 4,
                           csa.CSA_OUT_INDEX_FP8, _p(), 64, None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    r = L.csa_hca_compress(_p(), _p(), _p(), 512, 1, _p(), 256, _p(), 256, _p(), 4,
                           csa.CSA_OUT_KV_FP8, _p(), 64, None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    # HCA attention: negative or too many rows
    args = [_p(), 1, 64, _p(), _p(), csa.CSA_FMT_FP8, 64, 256, _p(), 4, _p(), 1, _p(), None, -1,
            128, 0.1, 1, _p(), None, _p(), 1 << 30, None, None]
    assert L.csa_hca_attention(*args) == csa.CSA_ERR_INVALID
    args[14] = csa.HCA_MAX_ROWS
    assert L.csa_hca_attention(*args) == csa.CSA_ERR_UNSUPPORTED
    # fused RoPE: odd or oversized rope_dim, no positions, rows_per_pos < 1, misaligned table
    def rope(rope_dim=64, positions=_p(), rows_per_pos=1, freqs=_p()):
        return L.csa_rope_hadamard_quant(_p(), csa.CSA_FMT_BF16, 4, 128, freqs, rope_dim, 1024,
                                         positions, rows_per_pos, csa.CSA_FMT_FP8, None, 0, _p(),
                                         None, _p(), None, None, None, None)
    assert rope(rope_dim=63) == csa.CSA_ERR_INVALID
    assert rope(rope_dim=130) == csa.CSA_ERR_INVALID
    assert rope(positions=None) == csa.CSA_ERR_INVALID
    assert rope(rows_per_pos=0) == csa.CSA_ERR_INVALID
    assert rope(freqs=ctypes.c_void_p(256 + 4)) == csa.CSA_ERR_INVALID
    r = L.csa_c4_compress_index_rope(_p(), _p(), _p(), 576, 1, _p(), 8, _p(), 8, _p(), 4,
                                     csa.CSA_OUT_KV_FP8, _p(), 64, 1024, _p(), None, None, 64,
                                     None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    # unrotated quantisation and the DSA calls share the C4 checks
    r = L.csa_index_quant(_p(), csa.CSA_FMT_BF16, 4, 96, csa.CSA_FMT_FP8, None, 0, _p(), None,
                          _p(), None, None, None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    r = L.csa_dsa_indexer_logits(_p(), None, _p(), 1, 64, 96, csa.CSA_FMT_FP8, _p(), None, _p(),
                                 64, _p(), 1, _p(), 1, _p(), None, 64, _p(), 64, None, None)
    assert r == csa.CSA_ERR_UNSUPPORTED
    r = L.csa_dsa_topk512_page_transform(_p(), 64, 1, _p(), 1, _p(), None, _p(), 4, 256, 32, 64,
                                         _p(), None, _p(), 1 << 20, None, None)
    assert r == csa.CSA_ERR_INVALID
    # fused indexer + top-512 with a workspace below its size
    r = L.csa_indexer_topk512(_p(), None, _p(), 1, 64, 128, csa.CSA_FMT_FP8, _p(), None, _p(), 64,
                              _p(), 1, _p(), 1, _p(), None, 64, 64, _p(), 64, _p(), None, _p(),
                              16, None, None)
    assert r == csa.CSA_ERR_WORKSPACE
    # the wait self-test needs a status word
    assert L.csa_selftest_wait_timeout(None, None, None) == csa.CSA_ERR_INVALID


def test_fp4_page_record_layout():
    """The test-side layout of CSA_FMT_FP4_PAGE records (include/csa.h) round
    trips and puts a hand-computed byte where the header says."""
    import numpy as np
    from gpu_util import fp4_page_records, fp4_page_unpack
    rng = np.random.default_rng(0)
    for dim in (64, 128):
        n = 128
        packed = rng.integers(0, 256, (n, dim // 2), dtype=np.uint8)
        bsc = rng.integers(0, 127, (n, dim // 16), dtype=np.uint8)
        sc = rng.uniform(0.1, 2.0, n).astype(np.float32)
        rec = fp4_page_records(packed, bsc, sc, dim)
        assert rec.shape == (2, 36 * dim + 256)
        pk, pb, ps = fp4_page_unpack(rec, dim)
        assert np.array_equal(pk, packed) and np.array_equal(pb, bsc) and np.array_equal(ps, sc)
        # key 73: page 1, r = 9, group 1, i = 1; groups of gb = 4.5*dim + 32 bytes
        gb = 4 * dim + dim // 2 + 32
        assert gb * 8 == 36 * dim + 256
        # code byte 17: gb + (17//16)*128 + 1*16 + 17%16
        assert rec[1, gb + 128 + 16 + 1] == packed[73, 17]
        # its second block scale and its row scale
        assert rec[1, gb + 4 * dim + dim // 16 + 1] == bsc[73, 1]
        o = gb + 4 * dim + dim // 2 + 4
        assert rec[1, o:o + 4].view(np.float32)[0] == sc[73]
