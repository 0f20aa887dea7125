"""Python face of the fp64 CPU oracle for C4 compressed sparse attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It wraps the plain C in
``csa_oracle.c`` (built with gcc, no fast-math) through ctypes and composes its
steps in the order the pages give them; it shares nothing with the CUDA
library in ``compressed_sparse_attention_12_b200``.

Pages cited (by title and section):
  [T] "Token 的一生：DSV4 架构与 DSpark" -- §1, §2.1, §2.2, §3.1, §3.2, §4
  [H] "DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）" -- "Compressed Sparse Attention（CSA）",
      "低精度與儲存策略的配合"
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

KV_DIM = 576
KV_LATENT = 512
KV_ROPE = 64
TOPK = 512
C4_RATIO = 4            # [T] §2.1: four raw tokens per compressed token
PAGE_SIZE = 256         # [T] §2.2: raw tokens per page
C4_PAGE_SIZE = PAGE_SIZE // C4_RATIO   # [T] §2.2: 64 compressed rows per page


def build(force: bool = False) -> str:
    """Compile csa_oracle.c into liboracle.so (gcc, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
           "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_L = ctypes.c_long
_I = ctypes.c_int
_D = ctypes.c_double


def _declare(L):
    L.oracle_e4m3_value.restype = _D
    L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    L.oracle_e2m1_value.restype = _D
    L.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
    L.oracle_ue4m3_value.restype = _D
    L.oracle_ue4m3_value.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_encode.restype = ctypes.c_uint8
    L.oracle_e4m3_encode.argtypes = [_D]
    L.oracle_e2m1_encode.restype = ctypes.c_uint8
    L.oracle_e2m1_encode.argtypes = [_D]
    L.oracle_ue4m3_encode.restype = ctypes.c_uint8
    L.oracle_ue4m3_encode.argtypes = [_D]
    L.oracle_bf16_encode.restype = ctypes.c_uint16
    L.oracle_bf16_encode.argtypes = [_D]
    L.oracle_bf16_encode_array.restype = None
    L.oracle_bf16_encode_array.argtypes = [_P, _L, _P]
    L.oracle_bf16_value.restype = _D
    L.oracle_bf16_value.argtypes = [ctypes.c_uint16]
    L.oracle_hadamard_matrix.restype = None
    L.oracle_hadamard_matrix.argtypes = [_I, _P]
    L.oracle_hadamard_rotate.restype = None
    L.oracle_hadamard_rotate.argtypes = [_P, _L, _I, _P]
    L.oracle_quant_fp8_rows.restype = None
    L.oracle_quant_fp8_rows.argtypes = [_P, _L, _I, _P, _P]
    L.oracle_quant_fp4_rows.restype = None
    L.oracle_quant_fp4_rows.argtypes = [_P, _L, _I, _P, _P, _P]
    L.oracle_dequant_fp8_rows.restype = None
    L.oracle_dequant_fp8_rows.argtypes = [_P, _P, _L, _I, _P]
    L.oracle_dequant_fp4_rows.restype = None
    L.oracle_dequant_fp4_rows.argtypes = [_P, _P, _P, _L, _I, _P]
    L.oracle_kv_encode_rows.restype = None
    L.oracle_kv_encode_rows.argtypes = [_P, _L, _I, _P]
    L.oracle_kv_decode_rows.restype = None
    L.oracle_kv_decode_rows.argtypes = [_P, _L, _I, _P]
    L.oracle_c4_compress.restype = _L
    L.oracle_c4_compress.argtypes = [_P, _P, _P, _L, _I, _P]
    L.oracle_pool_compress.restype = _L
    L.oracle_pool_compress.argtypes = [_P, _P, _P, _L, _I, _I, _P]
    L.oracle_indexer_logits.restype = None
    L.oracle_indexer_logits.argtypes = [_P, _P, _L, _I, _I, _P, _P, _P, _L]
    L.oracle_topk_transform.restype = _L
    L.oracle_topk_transform.argtypes = [_P, _L, _I, _P, _I, _L, _P, _P]
    L.oracle_sparse_attention.restype = None
    L.oracle_sparse_attention.argtypes = [_P, _I, _P, _L, _D, _P, _P]
    L.oracle_num_threads.restype = _I
    L.oracle_num_threads.argtypes = []
    L.oracle_set_num_threads.restype = None
    L.oracle_set_num_threads.argtypes = [_I]


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


# ---------------------------------------------------------------- formats

def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code) & 0xFF)


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code) & 0xF)


def ue4m3_value(code: int) -> float:
    return lib().oracle_ue4m3_value(int(code) & 0xFF)


def e4m3_encode(x: float) -> int:
    return lib().oracle_e4m3_encode(float(x))


def e2m1_encode(x: float) -> int:
    return lib().oracle_e2m1_encode(float(x))


def ue4m3_encode(x: float) -> int:
    return lib().oracle_ue4m3_encode(float(x))


def bf16_encode(x: float) -> int:
    return lib().oracle_bf16_encode(float(x))


def bf16_value(h: int) -> float:
    return lib().oracle_bf16_value(int(h) & 0xFFFF)


def e4m3_table() -> np.ndarray:
    """Value of every E4M3 byte (NaN for the two NaN codes)."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e2m1_table() -> np.ndarray:
    return np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def bf16_to_f64(h: np.ndarray) -> np.ndarray:
    """Decode raw bf16 bit patterns (uint16) to float64 (exact)."""
    h = np.asarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- Hadamard

def hadamard_matrix(n: int) -> np.ndarray:
    out = np.zeros((n, n), dtype=np.int8)
    lib().oracle_hadamard_matrix(n, _ptr(out))
    return out


def hadamard_rotate(x: np.ndarray) -> np.ndarray:
    """(1/sqrt(n)) H_n x over the last axis ([T] §4)."""
    x = _c(x, np.float64)
    n = x.shape[-1]
    rows = x.size // n
    y = np.empty_like(x)
    lib().oracle_hadamard_rotate(_ptr(x), rows, n, _ptr(y))
    return y


# ---------------------------------------------------------------- quantisers

def quant_fp8_rows(x: np.ndarray):
    """Per-row FP8 E4M3: returns (codes uint8 [..., n], scales float32 [...])."""
    x = _c(x, np.float64)
    n = x.shape[-1]
    rows = x.size // n
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty(x.shape[:-1], dtype=np.float32)
    lib().oracle_quant_fp8_rows(_ptr(x), rows, n, _ptr(codes), _ptr(scales))
    return codes, scales


def quant_fp4_rows(x: np.ndarray):
    """Per-row FP4 E2M1 with block-16 unsigned-E4M3 scales and a row fp32
    scale.  Returns (codes uint8 unpacked [..., n], block_scales uint8
    [..., n/16], row_scales float32 [...])."""
    x = _c(x, np.float64)
    n = x.shape[-1]
    assert n % 16 == 0
    rows = x.size // n
    codes = np.empty(x.shape, dtype=np.uint8)
    bsc = np.empty(x.shape[:-1] + (n // 16,), dtype=np.uint8)
    rsc = np.empty(x.shape[:-1], dtype=np.float32)
    lib().oracle_quant_fp4_rows(_ptr(x), rows, n, _ptr(codes), _ptr(bsc), _ptr(rsc))
    return codes, bsc, rsc


def dequant_fp8_rows(codes, scales) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    n = codes.shape[-1]
    out = np.empty(codes.shape, dtype=np.float64)
    lib().oracle_dequant_fp8_rows(_ptr(codes), _ptr(scales), codes.size // n, n, _ptr(out))
    return out


def dequant_fp4_rows(codes, block_scales, row_scales) -> np.ndarray:
    codes = _c(codes, np.uint8)
    block_scales = _c(block_scales, np.uint8)
    row_scales = _c(row_scales, np.float32)
    n = codes.shape[-1]
    out = np.empty(codes.shape, dtype=np.float64)
    lib().oracle_dequant_fp4_rows(_ptr(codes), _ptr(block_scales), _ptr(row_scales),
                                  codes.size // n, n, _ptr(out))
    return out


def pack_fp4(codes: np.ndarray) -> np.ndarray:
    """Two E2M1 codes per byte, element 2i in the low nibble, 2i+1 in the high
    nibble (the order of the packed FP4 index cache)."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] & 0xF) | ((codes[..., 1::2] & 0xF) << 4)


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def index_quantise(x: np.ndarray, fmt: str):
    """Rotation then quantisation of index queries/keys ([T] §3.1, §4).
    Returns a dict with the stored fields and the dequantised values."""
    return quantise_rows(hadamard_rotate(x), fmt)


def dsa_index_quantise(x: np.ndarray, fmt: str):
    """The DSA indexer's quantisation: the rows as given, no rotation ([T] §4:
    the Hadamard step is what DSV4 adds on top of DSA)."""
    return quantise_rows(x, fmt)


def rope(x: np.ndarray, freqs: np.ndarray, rope_dim: int, pos) -> np.ndarray:
    """Rotary embedding of the leading rope_dim values of each row ([T] §3.1
    freqs_cis / positions): the pairs (x[2i], x[2i+1]) read as complex numbers
    and multiplied by freqs[pos][i] = cos + i sin; the rest unchanged.
    x [..., D]; pos broadcasts against x.shape[:-1]; freqs [max_pos, rope_dim/2, 2]."""
    x = np.array(x, dtype=np.float64)
    f = np.asarray(freqs, dtype=np.float64)
    p = np.broadcast_to(np.asarray(pos, dtype=np.int64), x.shape[:-1])
    z = x[..., 0:rope_dim:2] + 1j * x[..., 1:rope_dim:2]
    rot = f[p, :, 0] + 1j * f[p, :, 1]
    y = z * rot
    x[..., 0:rope_dim:2] = y.real
    x[..., 1:rope_dim:2] = y.imag
    return x


def rope_index_quantise(x: np.ndarray, freqs: np.ndarray, rope_dim: int, pos, fmt: str):
    """[T] §3.1 / §4 fused order: RoPE, then the rotation, then quantisation."""
    return index_quantise(rope(x, freqs, rope_dim, pos), fmt)


def quantise_rows(xr: np.ndarray, fmt: str):
    """Quantisation of (already rotated or plain) index rows into `fmt`."""
    if fmt == "fp8":
        codes, scales = quant_fp8_rows(xr)
        return {"codes": codes, "scales": scales, "deq": dequant_fp8_rows(codes, scales)}
    if fmt == "fp4":
        codes, bsc, rsc = quant_fp4_rows(xr)
        return {"codes": codes, "packed": pack_fp4(codes), "block_scales": bsc,
                "scales": rsc, "deq": dequant_fp4_rows(codes, bsc, rsc)}
    if fmt == "bf16":
        h = bf16_encode_array(xr)
        return {"codes": h, "deq": bf16_to_f64(h)}
    raise ValueError(fmt)


def bf16_encode_array(x: np.ndarray) -> np.ndarray:
    """bf16 round-to-nearest-even of a float64 array (raw uint16 patterns)."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_bf16_encode_array(_ptr(x), x.size, _ptr(out))
    return out


# ---------------------------------------------------------------- KV rows

def kv_row_bytes(fp8: bool) -> int:
    return 656 if fp8 else 1152


def kv_encode_rows(x: np.ndarray, fp8: bool) -> np.ndarray:
    x = _c(x, np.float64).reshape(-1, KV_DIM)
    out = np.empty((x.shape[0], kv_row_bytes(fp8)), dtype=np.uint8)
    lib().oracle_kv_encode_rows(_ptr(x), x.shape[0], int(fp8), _ptr(out))
    return out


def kv_decode_rows(b: np.ndarray, fp8: bool) -> np.ndarray:
    b = _c(b, np.uint8).reshape(-1, kv_row_bytes(fp8))
    out = np.empty((b.shape[0], KV_DIM), dtype=np.float64)
    lib().oracle_kv_decode_rows(_ptr(b), b.shape[0], int(fp8), _ptr(out))
    return out


# ---------------------------------------------------------------- steps

def c4_compress(x: np.ndarray, gate: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """Step 1 ([T] §2.1): softmax-gated pooling of each complete block of 4
    raw rows; returns [floor(T/4), D]."""
    x = _c(x, np.float64)
    gate = _c(gate, np.float64)
    bias = _c(bias, np.float64)
    T, D = x.shape
    assert gate.shape == (T, D) and bias.shape == (4, D)
    y = np.empty((T // 4, D), dtype=np.float64)
    n = lib().oracle_c4_compress(_ptr(x), _ptr(gate), _ptr(bias), T, D, _ptr(y))
    assert n == T // 4
    return y


HCA_RATIO = 128         # [H] HCA: "about 128x" compression
HCA_PAGE_SIZE = PAGE_SIZE // HCA_RATIO   # compressed rows per 256-token page (reading)


def pool_compress(x: np.ndarray, gate: np.ndarray, bias: np.ndarray, ratio: int) -> np.ndarray:
    """Softmax-gated pooling over blocks of `ratio` raw rows with a per-position
    bias; the C4 compressor is ratio 4, the HCA compressor ([H] HCA) ratio 128.
    Returns [floor(T/ratio), D]."""
    x = _c(x, np.float64)
    gate = _c(gate, np.float64)
    bias = _c(bias, np.float64)
    T, D = x.shape
    assert gate.shape == (T, D) and bias.shape == (ratio, D)
    y = np.empty((T // ratio, D), dtype=np.float64)
    n = lib().oracle_pool_compress(_ptr(x), _ptr(gate), _ptr(bias), T, D, int(ratio), _ptr(y))
    assert n == T // ratio
    return y


def hca_compress(x: np.ndarray, gate: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """HCA compressor ([H] HCA): pool_compress with ratio 128."""
    return pool_compress(x, gate, bias, HCA_RATIO)


def hca_len(L: int) -> int:
    """HCA compressed length of a request with L raw tokens: floor(L/128)."""
    return L // HCA_RATIO


def hca_visible(pos: int) -> int:
    """HCA blocks visible to a query at raw position pos: floor((pos+1)/128)."""
    return (pos + 1) // HCA_RATIO


def hca_attention(q: np.ndarray, hca_rows: np.ndarray, window_rows: np.ndarray,
                  sm_scale: float):
    """HCA attention ([H] HCA: dense attention over the compressed blocks) for
    one query: every visible compressed row joined with the raw window rows
    under one softmax (the window is a reading: the pages describe it for CSA
    only; window 0 gives the compressed rows alone).  Returns (out [H, 512],
    lse [H])."""
    rows = np.concatenate([np.asarray(hca_rows, np.float64).reshape(-1, KV_DIM),
                           np.asarray(window_rows, np.float64).reshape(-1, KV_DIM)])
    return sparse_attention(q, rows, sm_scale)


def c4_len(L: int) -> int:
    """Compressed length of a request with L raw tokens ([T] §2.2): floor(L/4)."""
    return L // C4_RATIO


def n_visible(pos: int) -> int:
    """Compressed blocks visible to a query at raw position pos: those whose
    four tokens all lie at or before pos, i.e. floor((pos+1)/4)."""
    return (pos + 1) // C4_RATIO


def indexer_logits(q: np.ndarray, w: np.ndarray, k: np.ndarray, n_vis) -> np.ndarray:
    """Step 2: logits[t, s] = sum_h w[t,h] ReLU(q[t,h,:] . k[s,:]) for
    s < n_vis[t] (NaN elsewhere).  q [nq, Hi, Di], w [nq, Hi], k [n, Di]."""
    q = _c(q, np.float64)
    w = _c(w, np.float64)
    k = _c(k, np.float64)
    nq, Hi, Di = q.shape
    nv = _c(np.broadcast_to(np.asarray(n_vis), (nq,)), np.int64)
    assert nv.max(initial=0) <= k.shape[0]
    out = np.full((nq, k.shape[0]), np.nan, dtype=np.float64)
    lib().oracle_indexer_logits(_ptr(q), _ptr(w), nq, Hi, Di, _ptr(k), _ptr(nv), _ptr(out),
                                k.shape[0])
    return out


def topk_transform(logits_row: np.ndarray, n_vis: int, page_table_row: np.ndarray,
                   num_slots: int, k: int = TOPK, c4_page_size: int = C4_PAGE_SIZE):
    """Step 3 ([T] §3.2): (physical indices [k], logical indices [k]) with -1
    padding, selected in float on the row's first n_vis logits."""
    lg = _c(np.asarray(logits_row)[:n_vis], np.float32)
    assert not np.isnan(lg).any(), "NaN logits have no order"
    pt = _c(page_table_row, np.int32)
    phys = np.empty(k, dtype=np.int32)
    logical = np.empty(k, dtype=np.int32)
    r = lib().oracle_topk_transform(_ptr(lg), n_vis, k, _ptr(pt), c4_page_size, num_slots,
                                    _ptr(phys), _ptr(logical))
    if r < 0:
        raise IndexError("page table entry out of range")
    return phys, logical


def sparse_attention(q: np.ndarray, rows: np.ndarray, tau: float):
    """Step 4: one softmax over the given key rows (selected compressed rows and
    window rows together).  q [H, 576], rows [R, 576] -> (out [H, 512], lse [H])."""
    q = _c(q, np.float64)
    rows = _c(rows, np.float64).reshape(-1, KV_DIM)
    H = q.shape[0]
    out = np.empty((H, KV_LATENT), dtype=np.float64)
    lse = np.empty(H, dtype=np.float64)
    lib().oracle_sparse_attention(_ptr(q), H, _ptr(rows), rows.shape[0], float(tau),
                                  _ptr(out), _ptr(lse))
    return out, lse


def window_positions(pos: int, window: int) -> np.ndarray:
    """Raw positions in the sliding window of a query at raw position pos:
    [max(0, pos-window+1), pos] ([H] "Compressed Sparse Attention（CSA）")."""
    return np.arange(max(0, pos - window + 1), pos + 1, dtype=np.int64)


def raw_slot(page_table_row: np.ndarray, pos: np.ndarray, page_size: int = PAGE_SIZE):
    pos = np.asarray(pos, dtype=np.int64)
    return page_table_row[pos // page_size].astype(np.int64) * page_size + pos % page_size


# ---------------------------------------------------------------- whole step

def _t2n(x):
    """A torch tensor or numpy array as float64 numpy (exact for bf16/f32)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def step(w, data, page_table, requests=None, sm_scale=None, queries=None):
    """One decode/prefill step of C4 compressed sparse attention, composed from
    the steps above in the pages' order ([T] §1-§4; [H] "Compressed Sparse
    Attention（CSA）"), for the requests listed (default: all) and, within
    them, the query rows listed in `queries` (default: all).

    w is the workload's shape record and data its drawn inputs (the same
    buffers the GPU path reads).  The oracle keeps its own copies of the
    caches, quantised by its own codecs.  Returns a dict keyed by query row
    with the logical top-k indices, the logits, the output and the lse."""
    import math
    sm_scale = 1.0 / math.sqrt(KV_DIM) if sm_scale is None else sm_scale
    fp8_kv = w.kv_fmt == "fp8"
    bs = w.bs
    requests = range(bs) if requests is None else requests
    direct = np.asarray(w.direct_c4_lens)
    d_off = np.concatenate([[0], np.cumsum(direct)])
    n_off = np.asarray(w.cu_new)
    q_off = np.asarray(w.cu_q)
    q_pos = np.asarray(w.q_pos)
    raw_req = np.asarray(data["raw_req"])
    raw_pos = np.asarray(data["raw_pos"])
    out = {}
    for b in requests:
        L = int(w.seq_lens[b])
        # compressed rows: drawn directly, then the compressor's blocks ([T] §2.1)
        kv = _t2n(data["kv_c4"][d_off[b]:d_off[b + 1]])
        ik = _t2n(data["idx_k"][d_off[b]:d_off[b + 1]])
        if w.new_tokens[b] >= 4:
            sl = slice(n_off[b], n_off[b + 1])
            kv = np.concatenate([kv, c4_compress(_t2n(data["raw_kv"][sl]), _t2n(data["gate"][sl]),
                                                 _t2n(data["bias"]))])
            ik = np.concatenate([ik, c4_compress(_t2n(data["raw_idx_k"][sl]),
                                                 _t2n(data["idx_gate"][sl]),
                                                 _t2n(data["idx_bias"]))])
        n_c4 = c4_len(L)
        assert kv.shape[0] == n_c4 and ik.shape[0] == n_c4
        kv_deq = kv_decode_rows(kv_encode_rows(kv, fp8_kv), fp8_kv)
        k_deq = index_quantise(ik, w.idx_fmt)["deq"]
        # raw rows of this request, by position
        sel = raw_req == b
        raw_rows = dict(zip(raw_pos[sel].tolist(),
                            kv_decode_rows(kv_encode_rows(_t2n(data["kv_raw"][sel]), fp8_kv),
                                           fp8_kv)))
        rows_t = [t for t in range(int(q_off[b]), int(q_off[b + 1]))
                  if queries is None or t in queries]
        if not rows_t:
            continue
        qsel = np.asarray(rows_t, dtype=np.int64)
        qi = index_quantise(_t2n(data["q_idx"][qsel]), w.idx_fmt)["deq"]
        ww = _t2n(data["w"][qsel])
        pos = q_pos[qsel]
        nv = np.array([min(n_c4, n_visible(int(p))) for p in pos], dtype=np.int64)
        lg = indexer_logits(qi, ww, k_deq, nv) if n_c4 else np.zeros((len(pos), 0))
        qa = _t2n(data["q"][qsel])
        for j, p in enumerate(pos):
            t = rows_t[j]
            phys, logical = topk_transform(lg[j], int(nv[j]), page_table[b], 1 << 40, k=w.topk)
            chosen = logical[logical >= 0]
            win = window_positions(int(p), w.window)
            rows = np.concatenate([kv_deq[chosen].reshape(-1, KV_DIM),
                                   np.array([raw_rows[int(r)] for r in win]).reshape(-1, KV_DIM)])
            o, lse = sparse_attention(qa[j], rows, sm_scale)
            out[t] = {"logical": logical, "phys": phys, "logits": lg[j, :nv[j]], "out": o,
                      "lse": lse, "n_vis": int(nv[j])}
    return out


def hca_step(w, data, page_table, requests=None, sm_scale=None):
    """One HCA-layer step ([H] HCA: 128x compression, then dense attention over
    the compressed blocks) for the requests listed (default: all), from the
    same drawn buffers the GPU path reads (synth.draw_hca).

    Block j of request b (raw rows 128j .. 128j+127) is pooled by the
    compressor in this step when its last row is one of the step's query
    positions; earlier blocks arrive as drawn post-compression rows.  Each
    query at position p attends over the hca_visible(p) rows and its raw window
    under one softmax.  Returns a dict keyed by query row with out and lse."""
    import math
    sm_scale = 1.0 / math.sqrt(KV_DIM) if sm_scale is None else sm_scale
    fp8_kv = w.kv_fmt == "fp8"
    L_all = np.asarray(w.seq_lens, dtype=np.int64)
    Q_all = np.asarray(w.q_lens, dtype=np.int64)
    requests = range(len(L_all)) if requests is None else requests
    # which blocks each request's compressor pools in this step
    pooled = []
    for L, Q in zip(L_all, Q_all):
        js = [j for j in range(int(L) // HCA_RATIO) if int(L - Q) <= HCA_RATIO * j + HCA_RATIO - 1]
        pooled.append(js)
    n_direct = [hca_len(int(L)) - len(js) for L, js in zip(L_all, pooled)]
    d_off = np.concatenate([[0], np.cumsum(n_direct)]).astype(np.int64)
    n_off = np.concatenate([[0], np.cumsum([HCA_RATIO * len(js) for js in pooled])]).astype(np.int64)
    q_off = np.concatenate([[0], np.cumsum(Q_all)]).astype(np.int64)
    raw_req = np.asarray(data["raw_req"])
    raw_pos = np.asarray(data["raw_pos"])
    out = {}
    for b in requests:
        L, Q = int(L_all[b]), int(Q_all[b])
        rows = _t2n(data["hca_kv"][d_off[b]:d_off[b + 1]])
        if pooled[b]:
            sl = slice(n_off[b], n_off[b + 1])
            rows = np.concatenate([rows, hca_compress(_t2n(data["raw_kv"][sl]),
                                                      _t2n(data["gate"][sl]),
                                                      _t2n(data["bias"]))])
        assert rows.shape[0] == hca_len(L)
        deq = kv_decode_rows(kv_encode_rows(rows, fp8_kv), fp8_kv) if rows.shape[0] else rows
        sel = raw_req == b
        raw_rows = dict(zip(raw_pos[sel].tolist(),
                            kv_decode_rows(kv_encode_rows(_t2n(data["kv_raw"][sel]), fp8_kv),
                                           fp8_kv)))
        qa = _t2n(data["q"][q_off[b]:q_off[b + 1]])
        for j in range(Q):
            p = L - Q + j
            nv = min(hca_len(L), hca_visible(p))
            win = window_positions(p, w.window)
            wrows = np.array([raw_rows[int(r)] for r in win]).reshape(-1, KV_DIM)
            o, lse = hca_attention(qa[j], deq[:nv], wrows, sm_scale)
            out[int(q_off[b] + j)] = {"out": o, "lse": lse, "n_hca": nv}
    return out


def dsa_n_visible(pos: int) -> int:
    """Keys visible to a DSA query at raw position pos ([T] §1: one key per raw
    token, causal): the tokens 0..pos."""
    return pos + 1


def dsa_step(w, data, page_table, requests=None, sm_scale=None):
    """One DSA step ([T] §1: the indexer picks the top-k raw tokens, attention
    reads their KV) for the requests listed, k = 512: index keys and queries
    quantised without rotation, logits over keys s <= p, top-512 with the page
    transform of 64-token pages, one softmax over the selected raw rows (no
    window).  Returns a dict keyed by query row (logical, phys, out, lse)."""
    import math
    sm_scale = 1.0 / math.sqrt(KV_DIM) if sm_scale is None else sm_scale
    fp8_kv = w.kv_fmt == "fp8"
    L_all = np.asarray(w.seq_lens, dtype=np.int64)
    Q_all = np.asarray(w.q_lens, dtype=np.int64)
    requests = range(len(L_all)) if requests is None else requests
    l_off = np.concatenate([[0], np.cumsum(L_all)])
    q_off = np.concatenate([[0], np.cumsum(Q_all)])
    out = {}
    for b in requests:
        L, Q = int(L_all[b]), int(Q_all[b])
        keys = dsa_index_quantise(_t2n(data["idx_k"][l_off[b]:l_off[b + 1]]), w.idx_fmt)["deq"]
        qs = slice(q_off[b], q_off[b + 1])
        qi = dsa_index_quantise(_t2n(data["q_idx"][qs]), w.idx_fmt)["deq"]
        ww = _t2n(data["w"][qs])
        pos = np.arange(L - Q, L)
        nv = np.array([min(L, dsa_n_visible(int(p))) for p in pos], dtype=np.int64)
        lg = indexer_logits(qi, ww, keys, nv)
        kv_rows = _t2n(data["kv"][l_off[b]:l_off[b + 1]])
        qa = _t2n(data["q"][qs])
        for j, p in enumerate(pos):
            phys, logical = topk_transform(lg[j], int(nv[j]), page_table[b], 1 << 40, k=TOPK,
                                           c4_page_size=64)
            chosen = logical[logical >= 0]
            rows = kv_decode_rows(kv_encode_rows(kv_rows[chosen], fp8_kv), fp8_kv)
            o, lse = sparse_attention(qa[j], rows, sm_scale)
            out[int(q_off[b] + j)] = {"logical": logical, "phys": phys, "out": o, "lse": lse,
                                      "logits": lg[j, :nv[j]], "n_vis": int(nv[j])}
    return out
