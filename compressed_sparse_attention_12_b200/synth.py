"""Seeded synthetic workloads for C4 compressed sparse attention.

This module only draws random inputs and lays out page tables: it holds none
of the method's arithmetic (no pooling, rotation, quantisation, scoring,
selection or attention), so the CUDA library and the CPU oracle can both be
fed from the same buffers.

Every draw comes from a ``torch.Generator`` seeded from the workload's seed
and a fixed per-field stream number, on the device the caller names; the same
device and seed give the same bits.  Shapes follow the pages' workloads:
  - raw KV rows: 512 latent + 64 RoPE dims ([H] "低精度與儲存策略的配合"),
  - 4 raw tokens per compressed token ([T] §2.1), floor(L/4) compressed rows
    ([T] §2.2), pages of 256 raw / 64 compressed tokens ([T] §2.2),
  - top-512 selection ([T] §3.2), a sliding window of recent raw tokens
    ([H] "Compressed Sparse Attention（CSA）").
[T] = "Token 的一生：DSV4 架构与 DSpark"; [H] = "DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）".
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

KV_DIM = 576
PAGE_SIZE = 256
C4_PAGE = 64

# stream numbers: one independent generator per drawn field
_S_PAGES, _S_IDXK, _S_KVC4, _S_KVRAW, _S_QIDX, _S_W, _S_Q = 1, 2, 3, 4, 5, 6, 7
_S_RAWKV, _S_GATE, _S_BIAS, _S_RAWIK, _S_IGATE, _S_IBIAS, _S_LENS = 8, 9, 10, 11, 12, 13, 14
_S_HCA, _S_HGATE, _S_HBIAS = 15, 16, 17
_S_DSAK, _S_DSAKV, _S_FREQ = 18, 19, 20

# DSA comparison path: one index key per raw token, pages of 64 raw tokens
DSA_PAGE = 64

# HCA layers: 128 raw tokens per compressed row, 2 compressed rows per 256-token page
HCA_RATIO = 128
HCA_PAGE = PAGE_SIZE // HCA_RATIO


@dataclass
class Workload:
    """Shapes of one synthetic batch.

    seq_lens[b] is the raw length L of request b including its query tokens;
    its queries sit at raw positions L-q_lens[b] .. L-1.  The last
    new_tokens[b] raw rows of the request, starting on a block boundary, are
    handed to the compressor, which pools the complete blocks among them; the
    compressed rows before them are drawn directly as post-compression values.
    By default new_tokens covers exactly the blocks whose last token is one of
    this step's query tokens (a block is compressed when its fourth token
    arrives, [T] §2.1).
    """
    name: str
    seq_lens: np.ndarray
    q_lens: np.ndarray
    idx_heads: int
    idx_dim: int
    idx_fmt: str          # "bf16" | "fp8" | "fp4"
    heads: int
    kv_fmt: str           # "bf16" | "fp8"
    window: int = 128
    topk: int = 512
    key_dist: str = "normal"   # "normal" | "student_t3"
    new_tokens: np.ndarray | None = None
    seed: int = 0
    page_slack: int = 0   # extra unused pages in the pool (exercise the permutation)
    extra: dict = field(default_factory=dict)

    def __post_init__(self):
        self.seq_lens = np.asarray(self.seq_lens, dtype=np.int64)
        self.q_lens = np.asarray(self.q_lens, dtype=np.int64)
        assert (self.q_lens >= 1).all() and (self.q_lens <= self.seq_lens).all()
        if self.new_tokens is None:
            L, Q = self.seq_lens, self.q_lens
            j_min = -((-(L - Q - 3)) // 4)          # first block ending at a query position
            j_max = L // 4 - 1                       # last complete block
            start = np.where(j_min <= j_max, 4 * np.maximum(j_min, 0), L)
            self.new_tokens = L - start
        self.new_tokens = np.asarray(self.new_tokens, dtype=np.int64)
        assert (((self.seq_lens - self.new_tokens) % 4 == 0) | (self.new_tokens == 0)).all()
        assert (self.new_tokens >= 0).all() and (self.new_tokens <= self.seq_lens).all()

    @property
    def bs(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def c4_lens(self) -> np.ndarray:
        return self.seq_lens // 4

    @property
    def pages_per_req(self) -> np.ndarray:
        return (self.seq_lens + PAGE_SIZE - 1) // PAGE_SIZE

    @property
    def max_pages(self) -> int:
        return int(self.pages_per_req.max())

    @property
    def num_pages(self) -> int:
        return int(self.pages_per_req.sum()) + self.page_slack

    @property
    def num_q(self) -> int:
        return int(self.q_lens.sum())

    @property
    def cu_q(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int32)

    @property
    def q_pos(self) -> np.ndarray:
        """Raw position of every query token, request-major."""
        return np.concatenate([np.arange(L - q, L) for L, q in zip(self.seq_lens, self.q_lens)]
                              ).astype(np.int32)

    @property
    def q_req(self) -> np.ndarray:
        return np.repeat(np.arange(self.bs), self.q_lens).astype(np.int32)

    @property
    def compress_start(self) -> np.ndarray:
        """Raw position of the first row given to the compressor, per request."""
        return (self.seq_lens - self.new_tokens).astype(np.int64)

    @property
    def direct_c4_lens(self) -> np.ndarray:
        """Compressed rows drawn directly (those before the compressor's rows)."""
        return np.where(self.new_tokens > 0, self.compress_start // 4, self.c4_lens)

    @property
    def cu_new(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.new_tokens)]).astype(np.int32)

    def raw_window_start(self) -> np.ndarray:
        """First raw position whose row must be present in the raw cache: the
        window of the earliest query, and every row handed to the compressor."""
        first_q = self.seq_lens - self.q_lens
        return np.maximum(0, np.minimum(first_q - self.window + 1, self.compress_start))


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream * 7919) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def normal(shape, seed, stream, device, std=1.0, dtype=torch.float32, chunk_rows=1 << 20):
    """N(0, std^2) in float32, drawn in chunks of rows to bound peak memory."""
    g = _gen(seed, stream, device)
    out = torch.empty(shape, dtype=dtype, device=device)
    if out.numel() == 0:
        return out
    flat = out.view(shape[0], -1) if len(shape) > 1 else out.view(-1, 1)
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        t = torch.randn((r1 - r0, flat.shape[1]), generator=g, device=device, dtype=torch.float32)
        flat[r0:r1] = (t * std).to(dtype)
    return out


def student_t3(shape, seed, stream, device, chunk_rows=1 << 20):
    """Student-t with 3 degrees of freedom: z / sqrt(chi2_3 / 3)."""
    g = _gen(seed, stream, device)
    out = torch.empty(shape, dtype=torch.float32, device=device)
    if out.numel() == 0:
        return out
    flat = out.view(shape[0], -1)
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        n = (r1 - r0, flat.shape[1])
        z = torch.randn(n, generator=g, device=device)
        c = torch.randn((3,) + n, generator=g, device=device).square().sum(0)
        flat[r0:r1] = z / torch.sqrt(c / 3.0)
    return out


def uniform(shape, seed, stream, device):
    g = _gen(seed, stream, device)
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32)


def page_table(w: Workload) -> np.ndarray:
    """[bs, max_pages] int32: a seeded random permutation of the whole page pool
    hands each request its pages; unused entries are -1."""
    rng = np.random.default_rng(w.seed * 1_000_003 + _S_PAGES)
    perm = rng.permutation(w.num_pages).astype(np.int32)
    pt = np.full((w.bs, w.max_pages), -1, dtype=np.int32)
    o = 0
    for b, n in enumerate(w.pages_per_req):
        pt[b, :n] = perm[o:o + n]
        o += int(n)
    return pt


def draw(w: Workload, device="cpu", fields=None) -> dict:
    """Draw the workload's tensors on `device`.

    Returned fields (all row-major, request-major concatenation):
      idx_k     [sum direct_c4_lens, idx_dim] f32   index keys before rotation
      kv_c4     [sum direct_c4_lens, 576] f32        compressed KV rows
      raw_pos   [n_raw] int64 raw positions, raw_req [n_raw] int32 their request,
      kv_raw    [n_raw, 576] f32                     raw KV rows in the window
      q_idx     [num_q, idx_heads, idx_dim] bf16     index queries before rotation
      w         [num_q, idx_heads] f32 U(0,1)        head weights
      q         [num_q, heads, 576] bf16             attention queries
      raw_kv / gate [sum new_tokens, 576] f32, bias [4, 576] f32 ~N(0, 0.1^2);
                raw_kv is the slice of kv_raw at the compressor's positions
      raw_idx_k / idx_gate [sum new_tokens, idx_dim] f32, idx_bias [4, idx_dim]
    """
    want = (lambda f: True) if fields is None else (lambda f: f in fields)
    s = w.seed
    out = {}
    n_direct = int(w.direct_c4_lens.sum())
    if want("idx_k"):
        if w.key_dist == "student_t3":
            out["idx_k"] = student_t3((n_direct, w.idx_dim), s, _S_IDXK, device)
        else:
            out["idx_k"] = normal((n_direct, w.idx_dim), s, _S_IDXK, device)
    if want("kv_c4"):
        out["kv_c4"] = normal((n_direct, KV_DIM), s, _S_KVC4, device)
    need_raw = want("kv_raw") or want("raw_pos") or want("raw_kv")
    if need_raw:
        starts = w.raw_window_start()
        pos = np.concatenate([np.arange(a, L) for a, L in zip(starts, w.seq_lens)]).astype(np.int64)
        req = np.concatenate([np.full(L - a, b) for b, (a, L) in enumerate(zip(starts, w.seq_lens))]
                             ).astype(np.int32)
        out["raw_pos"] = pos
        out["raw_req"] = req
        out["kv_raw"] = normal((pos.shape[0], KV_DIM), s, _S_KVRAW, device)
    if want("q_idx"):
        out["q_idx"] = normal((w.num_q, w.idx_heads, w.idx_dim), s, _S_QIDX, device,
                              dtype=torch.bfloat16)
    if want("w"):
        out["w"] = uniform((w.num_q, w.idx_heads), s, _S_W, device)
    if want("q"):
        out["q"] = normal((w.num_q, w.heads, KV_DIM), s, _S_Q, device, dtype=torch.bfloat16)
    n_new = int(w.new_tokens.sum())
    if n_new and want("raw_kv"):
        # the compressor's raw rows are the raw-cache rows at [compress_start, L)
        sel = np.concatenate([np.nonzero((out["raw_req"] == b) & (out["raw_pos"] >= a))[0]
                              for b, a in enumerate(w.compress_start)])
        assert sel.shape[0] == n_new
        out["raw_kv"] = out["kv_raw"][torch.as_tensor(sel, device=out["kv_raw"].device)]
        out["gate"] = normal((n_new, KV_DIM), s, _S_GATE, device)
        out["bias"] = normal((4, KV_DIM), s, _S_BIAS, device, std=0.1)
    if n_new and want("raw_idx_k"):
        if w.key_dist == "student_t3":
            out["raw_idx_k"] = student_t3((n_new, w.idx_dim), s, _S_RAWIK, device)
        else:
            out["raw_idx_k"] = normal((n_new, w.idx_dim), s, _S_RAWIK, device)
        out["idx_gate"] = normal((n_new, w.idx_dim), s, _S_IGATE, device)
        out["idx_bias"] = normal((4, w.idx_dim), s, _S_IBIAS, device, std=0.1)
    return out


def ragged_lens(n: int, lo: int, hi: int, seed: int, short=(1234, 2047)) -> np.ndarray:
    """Raw lengths drawn log-uniform in [lo, hi]; the first len(short) requests
    get the given short lengths so that some compressed lengths fall below 512."""
    rng = np.random.default_rng(seed * 1_000_003 + _S_LENS)
    L = np.exp(rng.uniform(math.log(lo), math.log(hi), size=n)).astype(np.int64)
    L = np.clip(L, lo, hi)
    for i, v in enumerate(short[:n]):
        L[i] = v
    return L


def workload(name: str, scale: float = 1.0) -> Workload:
    """The synthetic workloads by name.  `scale` < 1 shrinks the context
    lengths (for oracle-sized parity runs) keeping every other shape."""
    def sc(L):
        return max(8, int(L * scale))
    if name == "tiny":
        # batch 1, 4096 raw tokens all compressed here, bf16 8x64 indexer, 16 heads, bf16 KV
        return Workload("tiny", [4096], [1], 8, 64, "bf16", 16, "bf16",
                        new_tokens=[4096], seed=0)
    if name == "decode_128k":
        # batch 32 x 131072, FP8 64x128 indexer, FP8 KV, 64 heads
        return Workload("decode_128k", [sc(131072)] * 32, [1] * 32, 64, 128, "fp8", 64, "fp8",
                        seed=1, page_slack=3)
    if name == "decode_1m":
        # batch 8 x 1048576, FP4 8x64 indexer (heavy-tailed keys), 16 heads, bf16 KV
        return Workload("decode_1m", [sc(1048576)] * 8, [1] * 8, 8, 64, "fp4", 16, "bf16",
                        key_dist="student_t3", seed=2, page_slack=3)
    if name == "decode_1m_wide":
        # as decode_1m with the 128K shapes: FP4 64x128 indexer, 64 heads, FP8 KV
        return Workload("decode_1m_wide", [sc(1048576)] * 8, [1] * 8, 64, 128, "fp4", 64, "fp8",
                        key_dist="student_t3", seed=2, page_slack=3)
    if name == "prefill":
        # 4096 new tokens appended to a 262144-token context; FP8 64x128 indexer
        ctx = sc(262144) // 4 * 4
        new = 4096 if scale >= 1.0 else max(8, min(4096, int(4096 * scale)) // 4 * 4)
        return Workload("prefill", [ctx + new], [new], 64, 128, "fp8", 64, "fp8",
                        seed=3, page_slack=1)
    if name == "dsa_128k":
        # DSA over raw tokens on the 128K decode shapes: FP8 64x128 indexer (not
        # rotated), 64 heads, FP8 KV, top-512 raw tokens, no window
        w = Workload("dsa_128k", [sc(131072)] * 32, [1] * 32, 64, 128, "fp8", 64, "fp8",
                     window=0, seed=5, page_slack=3, new_tokens=[0] * 32)
        return w
    if name.startswith("hca_"):
        # HCA layers ("DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", "Heavily Compressed
        # Attention（HCA）") on the shapes of the CSA workloads of the same size;
        # the indexer fields are unused
        base = {"hca_128k": "decode_128k", "hca_1m": "decode_1m",
                "hca_prefill": "prefill"}.get(name)
        if base is None:
            raise KeyError(name)
        w = workload(base, scale)
        w.name = name
        w.seed += 100
        return w
    if name == "ragged":
        # 64 requests, log-uniform lengths, Q alternating 1 / 5, FP4 indexer, FP8 KV
        L = ragged_lens(64, sc(2048), sc(1048576), seed=4,
                        short=(min(1234, sc(1234)), min(2047, sc(2047))))
        q = np.where(np.arange(64) % 2 == 0, 1, 5)
        return Workload("ragged", L, q, 64, 128, "fp4", 64, "fp8", seed=4, page_slack=5)
    raise KeyError(name)


def hca_plan(w: Workload):
    """HCA layer of the workload's requests: per request the raw position of
    the first row handed to the 128-row compressor (the blocks whose last token
    is one of this step's query tokens), how many raw rows it gets, and how
    many HCA rows before them are drawn directly as post-compression values."""
    L, Q = w.seq_lens, w.q_lens
    j_min = -((-(L - Q - (HCA_RATIO - 1))) // HCA_RATIO)
    j_max = L // HCA_RATIO - 1
    start = np.where(j_min <= j_max, HCA_RATIO * np.maximum(j_min, 0), L).astype(np.int64)
    new = (L - start).astype(np.int64)
    direct = np.where(new > 0, start // HCA_RATIO, L // HCA_RATIO).astype(np.int64)
    return start, new, direct


def draw_hca(w: Workload, device="cpu") -> dict:
    """Inputs of one HCA-layer step, on `device`:
      hca_kv  [sum direct, 576] f32     HCA rows drawn directly (before the compressor's)
      raw_pos [n_raw] int64, raw_req [n_raw] int32, kv_raw [n_raw, 576] f32
              raw rows from the earliest query's window or the compressor's
              first row, whichever is earlier, to L-1
      raw_kv / gate [sum new, 576] f32  the compressor's rows (slice of kv_raw) and gate
      bias    [128, 576] f32 ~N(0, 0.1^2)
      q       [num_q, heads, 576] bf16
    """
    s = w.seed
    start, new, direct = hca_plan(w)
    out = {"hca_kv": normal((int(direct.sum()), KV_DIM), s, _S_HCA, device)}
    first_q = w.seq_lens - w.q_lens
    lo = np.maximum(0, np.minimum(first_q - w.window + 1, start))
    pos = np.concatenate([np.arange(a, L) for a, L in zip(lo, w.seq_lens)]).astype(np.int64)
    req = np.concatenate([np.full(L - a, b) for b, (a, L) in enumerate(zip(lo, w.seq_lens))]
                         ).astype(np.int32)
    out["raw_pos"], out["raw_req"] = pos, req
    out["kv_raw"] = normal((pos.shape[0], KV_DIM), s, _S_KVRAW, device)
    n_new = int(new.sum())
    if n_new:
        sel = np.concatenate([np.nonzero((req == b) & (pos >= a))[0] for b, a in enumerate(start)])
        assert sel.shape[0] == n_new
        out["raw_kv"] = out["kv_raw"][torch.as_tensor(sel, device=out["kv_raw"].device)]
        out["gate"] = normal((n_new, KV_DIM), s, _S_HGATE, device)
        out["bias"] = normal((HCA_RATIO, KV_DIM), s, _S_HBIAS, device, std=0.1)
    out["q"] = normal((w.num_q, w.heads, KV_DIM), s, _S_Q, device, dtype=torch.bfloat16)
    return out


def dsa_page_table(w: Workload) -> np.ndarray:
    """[bs, max 64-token pages] int32: a seeded permutation of the pool of
    64-token pages; unused entries -1."""
    per = (w.seq_lens + DSA_PAGE - 1) // DSA_PAGE
    n = int(per.sum()) + w.page_slack
    rng = np.random.default_rng(w.seed * 1_000_003 + _S_PAGES)
    perm = rng.permutation(n).astype(np.int32)
    pt = np.full((w.bs, int(per.max())), -1, dtype=np.int32)
    o = 0
    for b, k in enumerate(per):
        pt[b, :k] = perm[o:o + k]
        o += int(k)
    return pt


def draw_dsa(w: Workload, device="cpu") -> dict:
    """Inputs of one DSA step, on `device` (every raw token has a KV row and an
    index key; this step's query tokens are the last q_lens[b] of each request
    and their rows are among them):
      idx_k  [sum L, idx_dim] f32   index keys of every raw token, request-major
      kv     [sum L, 576] f32       KV rows of every raw token
      q_idx  [num_q, idx_heads, idx_dim] bf16, w [num_q, idx_heads] f32 U(0,1),
      q      [num_q, heads, 576] bf16
    """
    s = w.seed
    n = int(w.seq_lens.sum())
    out = {"idx_k": normal((n, w.idx_dim), s, _S_DSAK, device),
           "kv": normal((n, KV_DIM), s, _S_DSAKV, device)}
    out["q_idx"] = normal((w.num_q, w.idx_heads, w.idx_dim), s, _S_QIDX, device,
                          dtype=torch.bfloat16)
    out["w"] = uniform((w.num_q, w.idx_heads), s, _S_W, device)
    out["q"] = normal((w.num_q, w.heads, KV_DIM), s, _S_Q, device, dtype=torch.bfloat16)
    return out


def rope_freqs(max_pos: int, rope_dim: int, base: float = 10000.0) -> torch.Tensor:
    """A rotary table [max_pos, rope_dim/2, 2] float32 of (cos, sin) of
    pos * base^(-2i/rope_dim), computed in float64 on the host.  An input of
    the fused RoPE kernels (the kernels never build it)."""
    i = np.arange(rope_dim // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / rope_dim)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * theta[None, :]
    return torch.from_numpy(np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32))
