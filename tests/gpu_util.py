"""Helpers for the GPU parity tests: lay out oracle-produced codes in the
library's array formats (a test-side marshalling step; the arithmetic
stays on each side) and compare results."""
import numpy as np
import torch

from oracle import oracle as orc


def dev(a):
    return torch.as_tensor(np.ascontiguousarray(a), device="cuda")


def code_bytes(fmt, dim):
    return {"bf16": 2 * dim, "fp8": dim, "fp4": dim // 2}[fmt]


def _fp4_page_offsets(dim):
    """Byte offsets inside a CSA_FMT_FP4_PAGE record (include/csa.h) of each
    key's code bytes [64, dim/2], block scales [64, dim/16] and row scale
    bytes [64, 4]."""
    gb = 4 * dim + dim // 2 + 32
    r = np.arange(64)[:, None]
    g, i = r // 8, r % 8
    b = np.arange(dim // 2)[None, :]
    codes = g * gb + (b // 16) * 128 + i * 16 + b % 16
    blocks = g * gb + 4 * dim + i * (dim // 16) + np.arange(dim // 16)[None, :]
    rows = g * gb + 4 * dim + dim // 2 + 4 * i + np.arange(4)[None, :]
    return codes, blocks, rows


def fp4_page_records(packed, bsc, sc, dim):
    """FP4 index arrays of n slots (n a multiple of 64) laid out as the
    paged records of CSA_FMT_FP4_PAGE: per 64-key page, 8 groups of 8 keys,
    each group's codes (8-key x 16-byte blocks), block scales and fp32 row
    scales side by side."""
    packed, bsc = np.asarray(packed, np.uint8), np.asarray(bsc, np.uint8)
    sc = np.asarray(sc, np.float32)
    n = packed.shape[0]
    assert n % 64 == 0
    pages = n // 64
    oc, ob, orow = _fp4_page_offsets(dim)
    rec = np.zeros((pages, 36 * dim + 256), dtype=np.uint8)
    rec[:, oc] = packed.reshape(pages, 64, dim // 2)
    rec[:, ob] = bsc.reshape(pages, 64, dim // 16)
    rec[:, orow] = sc.reshape(pages, 64).view(np.uint8).reshape(pages, 64, 4)
    return rec


def fp4_page_unpack(rec, dim):
    """Inverse of fp4_page_records: (packed codes, block scales, row scales)
    per slot."""
    rec = np.asarray(rec, np.uint8)
    pages = rec.shape[0]
    oc, ob, orow = _fp4_page_offsets(dim)
    packed = rec[:, oc].reshape(pages * 64, dim // 2)
    bsc = rec[:, ob].reshape(pages * 64, dim // 16)
    sc = np.ascontiguousarray(rec[:, orow]).view(np.float32).reshape(pages * 64)
    return packed, bsc, sc


def index_arrays(q, fmt, dim, n_rows, rows=None):
    """Oracle index quantisation result `q` (orc.index_quantise) written into
    [n_rows] library arrays at row indices `rows` (default 0..).  "fp4p": the
    FP4 result as paged records (keys; n_rows a multiple of 64), returned as
    (records, None, None)."""
    if fmt == "fp4p":
        codes, bsc, sc = (t.cpu().numpy() for t in index_arrays(q, "fp4", dim, n_rows, rows))
        return dev(fp4_page_records(codes, bsc, sc, dim)), None, None
    n = q["deq"].reshape(-1, dim).shape[0]
    rows = np.arange(n) if rows is None else np.asarray(rows)
    codes = np.zeros((n_rows, code_bytes(fmt, dim)), dtype=np.uint8)
    bsc = np.zeros((n_rows, dim // 16), dtype=np.uint8) if fmt == "fp4" else None
    sc = np.ones(n_rows, dtype=np.float32) if fmt != "bf16" else None
    if fmt == "bf16":
        codes[rows] = q["codes"].reshape(n, dim).astype(np.uint16).view(np.uint8).reshape(n, -1)
    elif fmt == "fp8":
        codes[rows] = q["codes"].reshape(n, dim)
        sc[rows] = q["scales"].reshape(n)
    else:
        codes[rows] = q["packed"].reshape(n, dim // 2)
        bsc[rows] = q["block_scales"].reshape(n, dim // 16)
        sc[rows] = q["scales"].reshape(n)
    return (dev(codes), dev(bsc) if bsc is not None else None,
            dev(sc) if sc is not None else None)


def decode_index_rows(codes, bsc, sc, fmt, dim):
    """Oracle-side decode of library index arrays (host numpy) to float64."""
    codes = np.asarray(codes)
    if fmt == "bf16":
        return orc.bf16_to_f64(codes.view(np.uint16).reshape(-1, dim))
    if fmt == "fp8":
        return orc.dequant_fp8_rows(codes, sc)
    return orc.dequant_fp4_rows(orc.unpack_fp4(codes), bsc, sc)


def code_values(codes, fmt, dim):
    """Per-element code values (no scales) of library arrays, float64."""
    codes = np.asarray(codes)
    if fmt == "bf16":
        return orc.bf16_to_f64(codes.view(np.uint16).reshape(-1, dim))
    if fmt == "fp8":
        return orc.e4m3_table()[codes]
    return orc.e2m1_table()[orc.unpack_fp4(codes)]


def rel_close(got, ref, rel, floor_frac=1e-3, axis=-1):
    """|got-ref| <= rel * max(|ref|, floor_frac * max|ref| along axis)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.maximum(np.abs(ref), floor_frac * np.abs(ref).max(axis=axis, keepdims=True))
    return np.abs(got - ref) <= rel * scale + 1e-30


def bf16_bound(ref, rel=2e-3, floor=None):
    """Error bound for a value computed in float32 and rounded once to bf16:
    the stated relative tolerance, or half a bf16 ulp of the reference where
    that is larger (2e-3 lies below bf16's half-ulp in the lower part of
    every binade, up to 2^-8 relative), plus an optional absolute term for
    the float32 error of the value before its rounding (cancellation)."""
    ref = np.abs(np.asarray(ref, dtype=np.float64))
    e = np.floor(np.log2(np.where(ref > 0, ref, 1.0)))
    half_ulp = np.where(ref > 0, 2.0 ** (e - 8), 0.0) * (1 + 2.0 ** -10)
    b = np.maximum(rel * ref, half_ulp)
    if floor is not None:
        b = b + floor    # float32 rounding before the bf16 rounding adds to it
    return b
