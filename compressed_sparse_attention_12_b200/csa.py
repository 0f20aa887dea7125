"""Thin ctypes binding of libcsa.so (include/csa.h), same names as the C ABI.

Argument marshalling only: every function takes torch tensors that already
live on the GPU (or plain ints/floats), passes their data pointers and the
current CUDA stream to the C entry point of the same name, and raises
``CsaError`` on a non-OK status.  Every step of the computation runs in the
library's CUDA kernels; if the library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_OK, CSA_ERR_INVALID, CSA_ERR_UNSUPPORTED, CSA_ERR_CUDA = 0, 1, 2, 3
CSA_ERR_TIMEOUT, CSA_ERR_BOUNDS, CSA_ERR_NAN, CSA_ERR_WORKSPACE = 4, 5, 6, 7
CSA_FMT_BF16, CSA_FMT_FP8, CSA_FMT_FP4, CSA_FMT_F32, CSA_FMT_FP4_PAGE = 0, 1, 2, 3, 4
CSA_OUT_KV_BF16, CSA_OUT_KV_FP8 = 0, 1
CSA_OUT_INDEX_BF16, CSA_OUT_INDEX_FP8, CSA_OUT_INDEX_FP4, CSA_OUT_INDEX_FP4_PAGE = 2, 3, 4, 5
TOPK, PAGE_SIZE, C4_PAGE_SIZE, KV_DIM, KV_LATENT = 512, 256, 64, 576, 512
TOPK_NOALLOC_MAX_BYTES = 16 << 20
HCA_RATIO, HCA_PAGE_SIZE, HCA_MAX_ROWS = 128, 2, 16 * 48 * 32

FMT = {"bf16": CSA_FMT_BF16, "fp8": CSA_FMT_FP8, "fp4": CSA_FMT_FP4, "fp4p": CSA_FMT_FP4_PAGE}


def index_record_bytes(dim: int) -> int:
    """Bytes of one CSA_FMT_FP4_PAGE record (the 64 keys of one page)."""
    return 36 * dim + 256


def _slots(fmt, codes):
    """Index slots held by a key array: one per row, 64 per paged FP4 record."""
    return codes.shape[0] * C4_PAGE_SIZE if fmt == CSA_FMT_FP4_PAGE else codes.shape[0]


class CsaError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn}: {status_string(code)} ({code})")


_lib = None
_P, _I32, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float

_SIGS = {
    "csa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "csa_abi_version": (_I32, []),
    "csa_kv_row_bytes": (_I32, [_I32]),
    "csa_kv_store": (ctypes.c_int, [_P, _I64, _P, _I32, _P, _I64, _P, _P]),
    "csa_c4_compress": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P, _I64, _P, _I32, _P, _I32,
                                       _I32, _P, _P, _P, _I64, _P, _P]),
    "csa_hadamard_quant": (ctypes.c_int, [_P, _I32, _I64, _I32, _I32, _P, _I64, _P, _P, _P,
                                          _P, _P, _P, _P]),
    "csa_indexer_logits": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _I64,
                                          _P, _I32, _P, _I32, _P, _P, _I32, _P, _I64, _P, _P]),
    "csa_topk512_workspace_size": (_SZ, [_I32, _I32]),
    "csa_topk512_page_transform": (ctypes.c_int, [_P, _I64, _I32, _P, _I32, _P, _P, _P, _I32,
                                                  _I64, _I32, _I32, _P, _P, _P, _SZ, _P, _P]),
    "csa_topk512_page_transform_noalloc": (ctypes.c_int, [_P, _I64, _I32, _P, _I32, _P, _P, _P,
                                                         _I32, _I64, _I32, _I32, _P, _P, _P,
                                                         _P]),
    "csa_indexer_topk512_workspace_size": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32]),
    "csa_indexer_topk512": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _I64,
                                           _P, _I32, _P, _I32, _P, _P, _I32, _I32, _P, _I64, _P,
                                           _P, _P, _SZ, _P, _P]),
    "csa_indexer_select": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _I64,
                                          _P, _I32, _P, _I32, _P, _P, _I32, _P, _I64, _P, _SZ,
                                          _P, _P]),
    "csa_topk512_merge": (ctypes.c_int, [_I32, _I32, _I32, _I32, _P, _I32, _P, _P, _P, _I32,
                                         _I64, _I32, _I32, _P, _P, _P, _SZ, _P, _P]),
    "csa_hca_compress": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P, _I64, _P, _I32, _P, _I32,
                                        _I32, _P, _I64, _P, _P]),
    "csa_hca_attention_workspace_size": (_SZ, [_I32, _I32, _I32, _I32, _I32]),
    "csa_hca_attention": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _I32, _I64, _I64, _P, _I32, _P,
                                         _I32, _P, _P, _I32, _I32, _F, _I32, _P, _P, _P, _SZ,
                                         _P, _P]),
    "csa_rope_hadamard_quant": (ctypes.c_int, [_P, _I32, _I64, _I32, _P, _I32, _I32, _P, _I32,
                                               _I32, _P, _I64, _P, _P, _P, _P, _P, _P, _P]),
    "csa_c4_compress_index_rope": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P, _I64, _P, _I32, _P,
                                                  _I32, _I32, _P, _I32, _I32, _P, _P, _P, _I64,
                                                  _P, _P]),
    "csa_index_quant": (ctypes.c_int, [_P, _I32, _I64, _I32, _I32, _P, _I64, _P, _P, _P, _P, _P,
                                       _P, _P]),
    "csa_dsa_indexer_logits": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P,
                                              _I64, _P, _I32, _P, _I32, _P, _P, _I32, _P, _I64,
                                              _P, _P]),
    "csa_dsa_topk512_page_transform": (ctypes.c_int, [_P, _I64, _I32, _P, _I32, _P, _P, _P, _I32,
                                                      _I64, _I32, _I32, _P, _P, _P, _SZ, _P,
                                                      _P]),
    "csa_sparse_mqa_workspace_size": (_SZ, [_I32, _I32, _I32, _I32]),
    "csa_workspace_size": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32]),
    "csa_selftest_wait_timeout": (ctypes.c_int, [_P, _P, _P]),
    "csa_sparse_mqa_decode": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _I32, _I64, _I64, _P, _P,
                                             _I32, _P, _I32, _P, _P, _I32, _F, _P, _P, _P, _SZ,
                                             _P, _P]),
    "csa_sparse_mqa_prefill": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _I32, _I64, _I64, _P, _P,
                                              _I32, _P, _I32, _P, _P, _I32, _F, _P, _P, _P, _SZ,
                                              _P, _P]),
}

EXPORTED = tuple(_SIGS)


def lib():
    """Load libcsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m compressed_sparse_attention_12_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().csa_status_string(int(code)).decode()


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libcsa takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libcsa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, code):
    if code != CSA_OK:
        raise CsaError(fn, code)


def csa_abi_version() -> int:
    return lib().csa_abi_version()


def csa_kv_row_bytes(kv_fmt: int) -> int:
    return lib().csa_kv_row_bytes(kv_fmt)


def csa_kv_store(rows, slots, kv_fmt, cache, status=None, stream=None):
    _check("csa_kv_store", lib().csa_kv_store(
        _ptr(rows), rows.shape[0], _ptr(slots), kv_fmt, _ptr(cache), cache.shape[0],
        _ptr(status), _stream(stream)))


def csa_c4_compress(x, gate, bias, cu_x, start_pos, max_rows_per_req, page_table, out_kind, out,
                    out_block_scales=None, out_scales=None, num_slots=None, status=None,
                    stream=None):
    bs = start_pos.shape[0]
    _check("csa_c4_compress", lib().csa_c4_compress(
        _ptr(x), _ptr(gate), _ptr(bias), x.shape[1], bs, _ptr(cu_x), x.shape[0], _ptr(start_pos),
        int(max_rows_per_req), _ptr(page_table), page_table.shape[1], out_kind, _ptr(out),
        _ptr(out_block_scales), _ptr(out_scales),
        _slots(CSA_FMT_FP4_PAGE if out_kind == CSA_OUT_INDEX_FP4_PAGE else -1, out)
        if num_slots is None else int(num_slots), _ptr(status), _stream(stream)))


def csa_hadamard_quant(x, fmt, codes, block_scales=None, scales=None, row_map=None,
                       w_in=None, w_out=None, status=None, stream=None):
    dim = x.shape[-1]
    rows = x.numel() // dim
    x_dtype = CSA_FMT_BF16 if x.dtype == torch.bfloat16 else CSA_FMT_F32
    n_out = _slots(fmt, codes) if row_map is not None else rows
    _check("csa_hadamard_quant", lib().csa_hadamard_quant(
        _ptr(x), x_dtype, rows, dim, fmt, _ptr(row_map), n_out, _ptr(codes), _ptr(block_scales),
        _ptr(scales), _ptr(w_in), _ptr(w_out), _ptr(status), _stream(stream)))


def csa_index_quant(x, fmt, codes, block_scales=None, scales=None, row_map=None,
                    w_in=None, w_out=None, status=None, stream=None):
    """Quantisation of index rows without the rotation (the DSA indexer)."""
    dim = x.shape[-1]
    rows = x.numel() // dim
    x_dtype = CSA_FMT_BF16 if x.dtype == torch.bfloat16 else CSA_FMT_F32
    n_out = _slots(fmt, codes) if row_map is not None else rows
    _check("csa_index_quant", lib().csa_index_quant(
        _ptr(x), x_dtype, rows, dim, fmt, _ptr(row_map), n_out, _ptr(codes), _ptr(block_scales),
        _ptr(scales), _ptr(w_in), _ptr(w_out), _ptr(status), _stream(stream)))


def csa_rope_hadamard_quant(x, freqs_cis, rope_dim, positions, rows_per_pos, fmt, codes,
                            block_scales=None, scales=None, row_map=None, w_in=None, w_out=None,
                            status=None, stream=None):
    """Rotary embedding, rotation and quantisation in one pass (include/csa.h).
    freqs_cis: [max_pos, rope_dim/2, 2] float32 (cos, sin)."""
    dim = x.shape[-1]
    rows = x.numel() // dim
    x_dtype = CSA_FMT_BF16 if x.dtype == torch.bfloat16 else CSA_FMT_F32
    n_out = _slots(fmt, codes) if row_map is not None else rows
    _check("csa_rope_hadamard_quant", lib().csa_rope_hadamard_quant(
        _ptr(x), x_dtype, rows, dim, _ptr(freqs_cis), int(rope_dim), freqs_cis.shape[0],
        _ptr(positions), int(rows_per_pos), fmt, _ptr(row_map), n_out, _ptr(codes),
        _ptr(block_scales), _ptr(scales), _ptr(w_in), _ptr(w_out), _ptr(status),
        _stream(stream)))


def csa_c4_compress_index_rope(x, gate, bias, cu_x, start_pos, max_rows_per_req, page_table,
                               out_kind, freqs_cis, rope_dim, out, out_block_scales=None,
                               out_scales=None, num_slots=None, status=None, stream=None):
    """C4 compressor in an index-key mode with the rotary embedding between the
    pooling and the rotation (include/csa.h)."""
    bs = start_pos.shape[0]
    _check("csa_c4_compress_index_rope", lib().csa_c4_compress_index_rope(
        _ptr(x), _ptr(gate), _ptr(bias), x.shape[1], bs, _ptr(cu_x), x.shape[0], _ptr(start_pos),
        int(max_rows_per_req), _ptr(page_table), page_table.shape[1], out_kind, _ptr(freqs_cis),
        int(rope_dim), freqs_cis.shape[0], _ptr(out), _ptr(out_block_scales), _ptr(out_scales),
        _slots(CSA_FMT_FP4_PAGE if out_kind == CSA_OUT_INDEX_FP4_PAGE else -1, out)
        if num_slots is None else int(num_slots), _ptr(status), _stream(stream)))


def csa_dsa_indexer_logits(q_codes, q_block_scales, q_weights, idx_heads, idx_dim, fmt, k_codes,
                           k_block_scales, k_scales, page_table, seq_lens, cu_q, q_pos,
                           max_seq_len, logits, num_slots=None, status=None, stream=None):
    """Indexer logits over raw tokens (one key per token, keys s <= p)."""
    num_q = q_weights.shape[0]
    _check("csa_dsa_indexer_logits", lib().csa_dsa_indexer_logits(
        _ptr(q_codes), _ptr(q_block_scales), _ptr(q_weights), num_q, idx_heads, idx_dim, fmt,
        _ptr(k_codes), _ptr(k_block_scales), _ptr(k_scales),
        _slots(fmt, k_codes) if num_slots is None else int(num_slots), _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], _ptr(cu_q), _ptr(q_pos),
        int(max_seq_len), _ptr(logits), logits.shape[1], _ptr(status), _stream(stream)))


def csa_dsa_topk512_page_transform(logits, seq_lens, cu_q, q_pos, page_table, num_slots,
                                   max_seq_len, out_indices, raw_indices=None, workspace=None,
                                   page_size=64, status=None, stream=None):
    """Top-512 over raw tokens with the 64-token page transform."""
    num_q = out_indices.shape[0]
    if workspace is None:
        workspace = torch.empty(max(1, csa_topk512_workspace_size(num_q, max_seq_len)),
                                dtype=torch.uint8, device=out_indices.device)
    _check("csa_dsa_topk512_page_transform", lib().csa_dsa_topk512_page_transform(
        _ptr(logits), logits.shape[1], num_q, _ptr(seq_lens), seq_lens.shape[0], _ptr(cu_q),
        _ptr(q_pos), _ptr(page_table), page_table.shape[1], int(num_slots), int(page_size),
        int(max_seq_len), _ptr(out_indices), _ptr(raw_indices), _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream)))


def csa_indexer_logits(q_codes, q_block_scales, q_weights, idx_heads, idx_dim, fmt, k_codes,
                       k_block_scales, k_scales, page_table, c4_seq_lens, cu_q, q_pos,
                       max_c4_len, logits, num_slots=None, status=None, stream=None):
    num_q = q_weights.shape[0]
    _check("csa_indexer_logits", lib().csa_indexer_logits(
        _ptr(q_codes), _ptr(q_block_scales), _ptr(q_weights), num_q, idx_heads, idx_dim, fmt,
        _ptr(k_codes), _ptr(k_block_scales), _ptr(k_scales),
        _slots(fmt, k_codes) if num_slots is None else int(num_slots), _ptr(page_table),
        page_table.shape[1], _ptr(c4_seq_lens), c4_seq_lens.shape[0], _ptr(cu_q), _ptr(q_pos),
        int(max_c4_len), _ptr(logits), logits.shape[1], _ptr(status), _stream(stream)))


def csa_topk512_workspace_size(num_q: int, max_c4_len: int) -> int:
    return lib().csa_topk512_workspace_size(num_q, max_c4_len)


def csa_topk512_page_transform(logits, c4_seq_lens, cu_q, q_pos, page_table, num_slots,
                               max_c4_len, out_indices, raw_indices=None, workspace=None,
                               c4_page_size=C4_PAGE_SIZE, status=None, stream=None):
    num_q = out_indices.shape[0]
    if workspace is None:
        workspace = torch.empty(max(1, csa_topk512_workspace_size(num_q, max_c4_len)),
                                dtype=torch.uint8, device=out_indices.device)
    _check("csa_topk512_page_transform", lib().csa_topk512_page_transform(
        _ptr(logits), logits.shape[1], num_q, _ptr(c4_seq_lens), c4_seq_lens.shape[0], _ptr(cu_q),
        _ptr(q_pos), _ptr(page_table), page_table.shape[1], int(num_slots), int(c4_page_size),
        int(max_c4_len), _ptr(out_indices), _ptr(raw_indices), _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream)))


def csa_topk512_page_transform_noalloc(logits, c4_seq_lens, cu_q, q_pos, page_table, num_slots,
                                       max_c4_len, out_indices, raw_indices=None,
                                       c4_page_size=C4_PAGE_SIZE, status=None, stream=None):
    """Top-512 page transform whose scratch is the library's own device array
    (no workspace, no allocation); see include/csa.h."""
    num_q = out_indices.shape[0]
    _check("csa_topk512_page_transform_noalloc", lib().csa_topk512_page_transform_noalloc(
        _ptr(logits), logits.shape[1], num_q, _ptr(c4_seq_lens), c4_seq_lens.shape[0], _ptr(cu_q),
        _ptr(q_pos), _ptr(page_table), page_table.shape[1], int(num_slots), int(c4_page_size),
        int(max_c4_len), _ptr(out_indices), _ptr(raw_indices), _ptr(status), _stream(stream)))


def csa_indexer_topk512_workspace_size(num_q, bs, idx_heads, idx_dim, fmt, max_c4_len) -> int:
    return lib().csa_indexer_topk512_workspace_size(num_q, bs, idx_heads, idx_dim, fmt,
                                                    max_c4_len)


def csa_indexer_topk512(q_codes, q_block_scales, q_weights, idx_heads, idx_dim, fmt, k_codes,
                        k_block_scales, k_scales, page_table, c4_seq_lens, cu_q, q_pos,
                        max_c4_len, logits, out_indices, raw_indices=None, workspace=None,
                        num_slots=None, c4_page_size=C4_PAGE_SIZE, status=None, stream=None):
    """Indexer logits + top-512 page transform in one call (see include/csa.h)."""
    num_q = q_weights.shape[0]
    bs = c4_seq_lens.shape[0]
    if workspace is None:
        n = csa_indexer_topk512_workspace_size(num_q, bs, idx_heads, idx_dim, fmt, max_c4_len)
        workspace = torch.empty(max(1, n), dtype=torch.uint8, device=logits.device)
    _check("csa_indexer_topk512", lib().csa_indexer_topk512(
        _ptr(q_codes), _ptr(q_block_scales), _ptr(q_weights), num_q, idx_heads, idx_dim, fmt,
        _ptr(k_codes), _ptr(k_block_scales), _ptr(k_scales),
        _slots(fmt, k_codes) if num_slots is None else int(num_slots), _ptr(page_table),
        page_table.shape[1], _ptr(c4_seq_lens), bs, _ptr(cu_q), _ptr(q_pos), int(max_c4_len),
        int(c4_page_size), _ptr(logits), logits.shape[1], _ptr(out_indices), _ptr(raw_indices),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)))


def csa_indexer_select(q_codes, q_block_scales, q_weights, idx_heads, idx_dim, fmt, k_codes,
                       k_block_scales, k_scales, page_table, c4_seq_lens, cu_q, q_pos,
                       max_c4_len, logits, workspace, num_slots=None, status=None, stream=None):
    """First half of csa_indexer_topk512: logits + per-chunk candidates."""
    num_q = q_weights.shape[0]
    _check("csa_indexer_select", lib().csa_indexer_select(
        _ptr(q_codes), _ptr(q_block_scales), _ptr(q_weights), num_q, idx_heads, idx_dim, fmt,
        _ptr(k_codes), _ptr(k_block_scales), _ptr(k_scales),
        _slots(fmt, k_codes) if num_slots is None else int(num_slots), _ptr(page_table),
        page_table.shape[1], _ptr(c4_seq_lens), c4_seq_lens.shape[0], _ptr(cu_q), _ptr(q_pos),
        int(max_c4_len), _ptr(logits), logits.shape[1], _ptr(workspace), workspace.numel(),
        _ptr(status), _stream(stream)))


def csa_topk512_merge(num_q, idx_heads, idx_dim, fmt, c4_seq_lens, cu_q, q_pos, page_table,
                      num_slots, max_c4_len, out_indices, workspace, raw_indices=None,
                      c4_page_size=C4_PAGE_SIZE, status=None, stream=None):
    """Second half of csa_indexer_topk512: row merge + page transform."""
    _check("csa_topk512_merge", lib().csa_topk512_merge(
        int(num_q), idx_heads, idx_dim, fmt, _ptr(c4_seq_lens), c4_seq_lens.shape[0], _ptr(cu_q),
        _ptr(q_pos), _ptr(page_table), page_table.shape[1], int(num_slots), int(c4_page_size),
        int(max_c4_len), _ptr(out_indices), _ptr(raw_indices), _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream)))


def csa_sparse_mqa_workspace_size(num_q, heads, window, decode) -> int:
    return lib().csa_sparse_mqa_workspace_size(num_q, heads, window, int(bool(decode)))


def _sparse_mqa(name, decode, q, c4_cache, raw_cache, kv_fmt, indices, page_table, seq_lens,
                cu_q, q_pos, window, sm_scale, out, lse=None, workspace=None, status=None,
                stream=None):
    num_q, heads = q.shape[0], q.shape[1]
    if workspace is None:
        n = csa_sparse_mqa_workspace_size(num_q, heads, window, decode)
        workspace = torch.empty(max(1, n), dtype=torch.uint8, device=q.device)
    fn = getattr(lib(), name)
    _check(name, fn(
        _ptr(q), num_q, heads, _ptr(c4_cache), _ptr(raw_cache), kv_fmt,
        c4_cache.shape[0] if c4_cache is not None else 0,
        raw_cache.shape[0] if raw_cache is not None else 0, _ptr(indices), _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], _ptr(cu_q), _ptr(q_pos),
        int(window), float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _ptr(status), _stream(stream)))


def csa_sparse_mqa_decode(*args, **kw):
    _sparse_mqa("csa_sparse_mqa_decode", True, *args, **kw)


def csa_sparse_mqa_prefill(*args, **kw):
    _sparse_mqa("csa_sparse_mqa_prefill", False, *args, **kw)


def csa_hca_compress(x, gate, bias, cu_x, start_pos, max_rows_per_req, page_table, out_kind, out,
                     num_slots=None, status=None, stream=None):
    """HCA compressor: softmax-gated pooling of blocks of 128 raw rows (see include/csa.h)."""
    bs = start_pos.shape[0]
    _check("csa_hca_compress", lib().csa_hca_compress(
        _ptr(x), _ptr(gate), _ptr(bias), x.shape[1], bs, _ptr(cu_x), x.shape[0], _ptr(start_pos),
        int(max_rows_per_req), _ptr(page_table), page_table.shape[1], out_kind, _ptr(out),
        out.shape[0] if num_slots is None else int(num_slots), _ptr(status), _stream(stream)))


def csa_hca_attention_workspace_size(num_q, heads, window, decode, max_hca_len) -> int:
    return lib().csa_hca_attention_workspace_size(num_q, heads, window, int(bool(decode)),
                                                  max_hca_len)


def csa_hca_attention(q, hca_cache, raw_cache, kv_fmt, page_table, seq_lens, cu_q, q_pos,
                      max_hca_len, window, sm_scale, decode, out, lse=None, workspace=None,
                      status=None, stream=None):
    """Dense attention over every visible HCA row plus the raw window (include/csa.h)."""
    num_q, heads = q.shape[0], q.shape[1]
    if workspace is None:
        n = csa_hca_attention_workspace_size(num_q, heads, window, decode, max_hca_len)
        workspace = torch.empty(max(1, n), dtype=torch.uint8, device=q.device)
    _check("csa_hca_attention", lib().csa_hca_attention(
        _ptr(q), num_q, heads, _ptr(hca_cache), _ptr(raw_cache), kv_fmt,
        hca_cache.shape[0] if hca_cache is not None else 0,
        raw_cache.shape[0] if raw_cache is not None else 0, _ptr(page_table), page_table.shape[1],
        _ptr(seq_lens), seq_lens.shape[0], _ptr(cu_q), _ptr(q_pos), int(max_hca_len),
        int(window), float(sm_scale), int(bool(decode)), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream)))


CSA_OP_TOPK512, CSA_OP_INDEXER_TOPK512, CSA_OP_SPARSE_MQA, CSA_OP_HCA_ATTENTION = 1, 2, 3, 4


def csa_workspace_size(op, bs=0, max_rows=0, max_len=0, heads=0, window=0, decode=True,
                       idx_dim=0, fmt=0) -> int:
    """Workspace bytes of one operation by code (include/csa.h)."""
    return lib().csa_workspace_size(op, bs, max_rows, max_len, heads, window, int(bool(decode)),
                                    idx_dim, fmt)


def csa_selftest_wait_timeout(status, waited_ns=None, stream=None):
    """One bounded device wait that runs out (include/csa.h)."""
    _check("csa_selftest_wait_timeout", lib().csa_selftest_wait_timeout(
        _ptr(status), _ptr(waited_ns), _stream(stream)))
