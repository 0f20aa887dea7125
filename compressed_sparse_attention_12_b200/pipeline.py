"""One C4 compressed-sparse-attention step on the GPU, through libcsa only.

``CsaBatch`` owns the paged device caches of a workload (compressed KV rows,
raw KV rows, index keys) and the per-step buffers; ``step()`` runs the four
steps of the pages in order ("Token 的一生：DSV4 架构与 DSpark" §1-§3;
"DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", "Compressed Sparse Attention（CSA）"):

  1. c4 compress of the blocks completed by this step's tokens (KV rows and
     index keys),
  2. rotation + quantisation of the index queries, then the indexer logits,
  3. top-512 with the page transform,
  4. sparse attention over the 512 rows plus the sliding window.

Everything that computes runs in libcsa's kernels; this module only sizes
and fills buffers (the cache contents come from the workload's drawn rows,
written by the library's own store/quantise/compress kernels).
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import csa
from .synth import Workload, page_table as make_page_table

PAGE, C4P = 256, 64


def code_bytes(fmt: str, dim: int) -> int:
    return {"bf16": 2 * dim, "fp8": dim, "fp4": dim // 2}[fmt]


def c4_slots(pt: np.ndarray, b: int, s: np.ndarray) -> np.ndarray:
    return pt[b, s // C4P].astype(np.int64) * C4P + s % C4P


def raw_slots(pt: np.ndarray, b: int, r: np.ndarray) -> np.ndarray:
    return pt[b, r // PAGE].astype(np.int64) * PAGE + r % PAGE


class CsaBatch:
    def __init__(self, w: Workload, data: dict, device="cuda", sm_scale=None, paged_fp4=False):
        self.w = w
        self.device = device
        dev = device
        self.kv_fmt = csa.FMT[w.kv_fmt]
        self.idx_fmt = csa.FMT[w.idx_fmt]
        self.sm_scale = float(sm_scale if sm_scale is not None else 1.0 / math.sqrt(csa.KV_DIM))
        pt = make_page_table(w)
        self.pt_host = pt
        self.page_table = torch.as_tensor(pt, device=dev)
        self.num_pages = w.num_pages
        self.c4_slots_n = self.num_pages * C4P
        self.raw_slots_n = self.num_pages * PAGE
        rb = csa.csa_kv_row_bytes(self.kv_fmt)
        self.c4_cache = torch.zeros((self.c4_slots_n, rb), dtype=torch.uint8, device=dev)
        self.raw_cache = torch.zeros((self.raw_slots_n, rb), dtype=torch.uint8, device=dev)
        Di, Hi = w.idx_dim, w.idx_heads
        cb = code_bytes(w.idx_fmt, Di)
        # index keys: structure of arrays (codes, FP4 block scales, row scales);
        # paged_fp4=True keeps FP4 keys as one CSA_FMT_FP4_PAGE record per page
        self.key_fmt = csa.CSA_FMT_FP4_PAGE if (paged_fp4 and w.idx_fmt == "fp4") else self.idx_fmt
        if self.key_fmt == csa.CSA_FMT_FP4_PAGE:
            self.k_codes = torch.zeros((self.num_pages, csa.index_record_bytes(Di)),
                                       dtype=torch.uint8, device=dev)
            self.k_bsc = self.k_scales = None
        else:
            self.k_codes = torch.zeros((self.c4_slots_n, cb), dtype=torch.uint8, device=dev)
            self.k_bsc = (torch.zeros((self.c4_slots_n, Di // 16), dtype=torch.uint8, device=dev)
                          if w.idx_fmt == "fp4" else None)
            self.k_scales = (torch.ones(self.c4_slots_n, dtype=torch.float32, device=dev)
                             if w.idx_fmt != "bf16" else None)
        i32 = lambda a: torch.as_tensor(np.asarray(a, dtype=np.int32), device=dev)
        self.seq_lens = i32(w.seq_lens)
        self.c4_lens = i32(w.c4_lens)
        self.cu_q = i32(w.cu_q)
        self.q_pos = i32(w.q_pos)
        self.cu_new = i32(w.cu_new)
        self.start_pos = i32(w.compress_start)
        self.max_new = int(w.new_tokens.max()) if w.bs else 0
        self.max_c4 = int(w.c4_lens.max())
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

        # --- fill the caches from the drawn rows (library kernels do the formatting)
        direct = w.direct_c4_lens
        slots = np.concatenate([c4_slots(pt, b, np.arange(n)) for b, n in enumerate(direct)]
                               ) if direct.sum() else np.zeros(0, np.int64)
        slots_t = i32(slots)
        if slots.size:
            csa.csa_kv_store(data["kv_c4"].contiguous(), slots_t, self.kv_fmt, self.c4_cache,
                             status=self.status)
            csa.csa_hadamard_quant(data["idx_k"].contiguous(), self.key_fmt, self.k_codes,
                                   self.k_bsc, self.k_scales, row_map=slots_t, status=self.status)
        rreq, rpos = np.asarray(data["raw_req"]), np.asarray(data["raw_pos"])
        rs = pt[rreq, rpos // PAGE].astype(np.int64) * PAGE + rpos % PAGE
        self.raw_slot_list = rs
        if rs.size:
            csa.csa_kv_store(data["kv_raw"].contiguous(), i32(rs), self.kv_fmt, self.raw_cache,
                             status=self.status)

        # --- per-step inputs
        self.raw_kv = data.get("raw_kv")
        self.gate = data.get("gate")
        self.bias = data.get("bias")
        self.raw_idx_k = data.get("raw_idx_k")
        self.idx_gate = data.get("idx_gate")
        self.idx_bias = data.get("idx_bias")
        self.q_idx = data["q_idx"].contiguous()
        self.w_head = data["w"].contiguous()
        self.q = data["q"].contiguous()

        nq = w.num_q
        self.q_codes = torch.empty((nq * Hi, cb), dtype=torch.uint8, device=dev)
        self.q_bsc = (torch.empty((nq * Hi, Di // 16), dtype=torch.uint8, device=dev)
                      if w.idx_fmt == "fp4" else None)
        self.q_scales = torch.empty(nq * Hi, dtype=torch.float32, device=dev)
        self.w_fold = torch.empty((nq, Hi), dtype=torch.float32, device=dev)
        self.logit_stride = max(16, (self.max_c4 + 15) // 16 * 16)
        self.logits = torch.empty((nq, self.logit_stride), dtype=torch.float32, device=dev)
        self.indices = torch.empty((nq, csa.TOPK), dtype=torch.int32, device=dev)
        self.raw_indices = torch.empty((nq, csa.TOPK), dtype=torch.int32, device=dev)
        self.topk_ws = torch.empty(max(1, csa.csa_topk512_workspace_size(nq, self.max_c4)),
                                   dtype=torch.uint8, device=dev)
        self.fused_ws = torch.empty(
            max(1, csa.csa_indexer_topk512_workspace_size(nq, w.bs, w.idx_heads, w.idx_dim,
                                                          self.key_fmt, self.max_c4)),
            dtype=torch.uint8, device=dev)
        self.decode = bool((w.q_lens <= 8).all())
        self.attn_ws = torch.empty(
            max(1, csa.csa_sparse_mqa_workspace_size(nq, w.heads, w.window, self.decode)),
            dtype=torch.uint8, device=dev)
        self.out = torch.empty((nq, w.heads, csa.KV_LATENT), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((nq, w.heads), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        self.check_status()

    def check_status(self):
        s = int(self.status.item())
        if s != 0:
            raise csa.CsaError("device status", s)

    # ------------------------------------------------------------------ steps
    def compress(self, stream=None):
        self.compress_kv(stream)
        self.compress_index(stream)

    def compress_kv(self, stream=None):
        """The compressor over this step's completed blocks, KV rows."""
        w = self.w
        if self.max_new < 4 or self.raw_kv is None:
            return
        kv_kind = csa.CSA_OUT_KV_FP8 if w.kv_fmt == "fp8" else csa.CSA_OUT_KV_BF16
        csa.csa_c4_compress(self.raw_kv, self.gate, self.bias, self.cu_new, self.start_pos,
                            self.max_new, self.page_table, kv_kind, self.c4_cache,
                            status=self.status, stream=stream)

    def compress_index(self, stream=None):
        """The compressor over this step's completed blocks, index keys."""
        w = self.w
        if self.max_new < 4 or self.raw_idx_k is None:
            return
        ik = {"bf16": csa.CSA_OUT_INDEX_BF16, "fp8": csa.CSA_OUT_INDEX_FP8,
              "fp4": csa.CSA_OUT_INDEX_FP4}[w.idx_fmt]
        if self.key_fmt == csa.CSA_FMT_FP4_PAGE:
            ik = csa.CSA_OUT_INDEX_FP4_PAGE
        csa.csa_c4_compress(self.raw_idx_k, self.idx_gate, self.idx_bias, self.cu_new,
                            self.start_pos, self.max_new, self.page_table, ik, self.k_codes,
                            self.k_bsc, self.k_scales, status=self.status, stream=stream)

    def index(self, stream=None):
        w = self.w
        csa.csa_hadamard_quant(self.q_idx, self.idx_fmt, self.q_codes, self.q_bsc, self.q_scales,
                               w_in=self.w_head, w_out=self.w_fold, status=self.status,
                               stream=stream)
        csa.csa_indexer_logits(self.q_codes, self.q_bsc, self.w_fold, w.idx_heads, w.idx_dim,
                               self.key_fmt, self.k_codes, self.k_bsc, self.k_scales,
                               self.page_table, self.c4_lens, self.cu_q, self.q_pos, self.max_c4,
                               self.logits, status=self.status, stream=stream)

    def quantise_q(self, stream=None):
        csa.csa_hadamard_quant(self.q_idx, self.idx_fmt, self.q_codes, self.q_bsc, self.q_scales,
                               w_in=self.w_head, w_out=self.w_fold, status=self.status,
                               stream=stream)

    def index_select(self, stream=None):
        """Indexer logits and top-512 in one call (the indexer CTAs select their
        own chunks; see csa_indexer_topk512)."""
        w = self.w
        self.quantise_q(stream)
        csa.csa_indexer_topk512(self.q_codes, self.q_bsc, self.w_fold, w.idx_heads, w.idx_dim,
                                self.key_fmt, self.k_codes, self.k_bsc, self.k_scales,
                                self.page_table, self.c4_lens, self.cu_q, self.q_pos, self.max_c4,
                                self.logits, self.indices, self.raw_indices, self.fused_ws,
                                num_slots=self.c4_slots_n, status=self.status, stream=stream)

    def select(self, stream=None):
        csa.csa_topk512_page_transform(self.logits, self.c4_lens, self.cu_q, self.q_pos,
                                       self.page_table, self.c4_slots_n, self.max_c4,
                                       self.indices, self.raw_indices, self.topk_ws,
                                       status=self.status, stream=stream)

    def attend(self, stream=None):
        fn = csa.csa_sparse_mqa_decode if self.decode else csa.csa_sparse_mqa_prefill
        fn(self.q, self.c4_cache, self.raw_cache, self.kv_fmt, self.indices, self.page_table,
           self.seq_lens, self.cu_q, self.q_pos, self.w.window, self.sm_scale, self.out,
           self.lse, self.attn_ws, status=self.status, stream=stream)

    def step(self, stream=None, fused=True):
        self.compress(stream)
        if fused:
            self.index_select(stream)
        else:
            self.index(stream)
            self.select(stream)
        self.attend(stream)
        return self.out


def hca_slots(pt: np.ndarray, b: int, j: np.ndarray) -> np.ndarray:
    """HCA slot of compressed row j of request b: page p of the HCA cache holds
    the 2 compressed rows of raw page p."""
    return pt[b, j // csa.HCA_PAGE_SIZE].astype(np.int64) * csa.HCA_PAGE_SIZE + \
        j % csa.HCA_PAGE_SIZE


class HcaBatch:
    """One HCA-layer step ("DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", "Heavily
    Compressed Attention（HCA）"): the 128-row compressor over the blocks
    completed by this step's tokens, then dense attention of every query over
    all visible HCA rows plus the raw window.  Same paging as CsaBatch: one page
    table serves the raw cache (256 rows per page) and the HCA cache (2 rows
    per page)."""

    def __init__(self, w: Workload, data: dict, device="cuda", sm_scale=None):
        from .synth import hca_plan
        self.w = w
        self.device = device
        dev = device
        self.kv_fmt = csa.FMT[w.kv_fmt]
        self.sm_scale = float(sm_scale if sm_scale is not None else 1.0 / math.sqrt(csa.KV_DIM))
        pt = make_page_table(w)
        self.pt_host = pt
        self.page_table = torch.as_tensor(pt, device=dev)
        self.num_pages = w.num_pages
        self.hca_slots_n = self.num_pages * csa.HCA_PAGE_SIZE
        self.raw_slots_n = self.num_pages * PAGE
        rb = csa.csa_kv_row_bytes(self.kv_fmt)
        self.hca_cache = torch.zeros((self.hca_slots_n, rb), dtype=torch.uint8, device=dev)
        self.raw_cache = torch.zeros((self.raw_slots_n, rb), dtype=torch.uint8, device=dev)
        start, new, direct = hca_plan(w)
        i32 = lambda a: torch.as_tensor(np.asarray(a, dtype=np.int32), device=dev)
        self.seq_lens = i32(w.seq_lens)
        self.cu_q = i32(w.cu_q)
        self.q_pos = i32(w.q_pos)
        self.start_pos = i32(start)
        self.cu_new = i32(np.concatenate([[0], np.cumsum(new)]))
        self.new_tokens = new
        self.max_new = int(new.max()) if w.bs else 0
        self.max_hca = int((w.seq_lens // csa.HCA_RATIO).max())
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        slots = np.concatenate([hca_slots(pt, b, np.arange(n)) for b, n in enumerate(direct)]
                               ) if direct.sum() else np.zeros(0, np.int64)
        if slots.size:
            csa.csa_kv_store(data["hca_kv"].contiguous(), i32(slots), self.kv_fmt, self.hca_cache,
                             status=self.status)
        rreq, rpos = np.asarray(data["raw_req"]), np.asarray(data["raw_pos"])
        rs = pt[rreq, rpos // PAGE].astype(np.int64) * PAGE + rpos % PAGE
        if rs.size:
            csa.csa_kv_store(data["kv_raw"].contiguous(), i32(rs), self.kv_fmt, self.raw_cache,
                             status=self.status)
        self.raw_kv = data.get("raw_kv")
        self.gate = data.get("gate")
        self.bias = data.get("bias")
        self.q = data["q"].contiguous()
        nq = w.num_q
        self.decode = bool((w.q_lens <= 8).all())
        self.attn_ws = torch.empty(
            max(1, csa.csa_hca_attention_workspace_size(nq, w.heads, w.window, self.decode,
                                                        self.max_hca)),
            dtype=torch.uint8, device=dev)
        self.out = torch.empty((nq, w.heads, csa.KV_LATENT), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((nq, w.heads), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        self.check_status()

    def check_status(self):
        s = int(self.status.item())
        if s != 0:
            raise csa.CsaError("device status", s)

    def compress(self, stream=None):
        if self.max_new < csa.HCA_RATIO or self.raw_kv is None:
            return
        kind = csa.CSA_OUT_KV_FP8 if self.w.kv_fmt == "fp8" else csa.CSA_OUT_KV_BF16
        csa.csa_hca_compress(self.raw_kv, self.gate, self.bias, self.cu_new, self.start_pos,
                             self.max_new, self.page_table, kind, self.hca_cache,
                             num_slots=self.hca_slots_n, status=self.status, stream=stream)

    def attend(self, stream=None):
        csa.csa_hca_attention(self.q, self.hca_cache, self.raw_cache, self.kv_fmt, self.page_table,
                              self.seq_lens, self.cu_q, self.q_pos, self.max_hca, self.w.window,
                              self.sm_scale, self.decode, self.out, self.lse, self.attn_ws,
                              status=self.status, stream=stream)

    def step(self, stream=None):
        self.compress(stream)
        self.attend(stream)
        return self.out


class DsaBatch:
    """One step of the DSA comparison path ("Token 的一生：DSV4 架构与 DSpark" §1
    从 DSA 到 DSV4): the indexer scores every raw token, the top-512 raw
    tokens are attended to.  One page table of 64-token pages serves the KV
    cache and the index K cache.  The step: store this step's tokens (KV row,
    plain-quantised index key), quantise the index queries (no rotation),
    indexer logits over keys s <= p, top-512 page transform, attention over the
    selected raw rows (no window)."""

    def __init__(self, w: Workload, data: dict, device="cuda", sm_scale=None):
        from .synth import DSA_PAGE, dsa_page_table
        self.w = w
        dev = device
        self.kv_fmt = csa.FMT[w.kv_fmt]
        self.idx_fmt = csa.FMT[w.idx_fmt]
        self.sm_scale = float(sm_scale if sm_scale is not None else 1.0 / math.sqrt(csa.KV_DIM))
        pt = dsa_page_table(w)
        self.pt_host = pt
        self.page_table = torch.as_tensor(pt, device=dev)
        per = (w.seq_lens + DSA_PAGE - 1) // DSA_PAGE
        self.slots_n = (int(per.sum()) + w.page_slack) * DSA_PAGE
        rb = csa.csa_kv_row_bytes(self.kv_fmt)
        Di, Hi = w.idx_dim, w.idx_heads
        cb = code_bytes(w.idx_fmt, Di)
        self.kv_cache = torch.zeros((self.slots_n, rb), dtype=torch.uint8, device=dev)
        self.k_codes = torch.zeros((self.slots_n, cb), dtype=torch.uint8, device=dev)
        self.k_bsc = (torch.zeros((self.slots_n, Di // 16), dtype=torch.uint8, device=dev)
                      if w.idx_fmt == "fp4" else None)
        self.k_scales = (torch.ones(self.slots_n, dtype=torch.float32, device=dev)
                         if w.idx_fmt != "bf16" else None)
        i32 = lambda a: torch.as_tensor(np.asarray(a, dtype=np.int32), device=dev)
        self.seq_lens = i32(w.seq_lens)
        self.cu_q = i32(w.cu_q)
        self.q_pos = i32(w.q_pos)
        self.max_len = int(w.seq_lens.max())
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        # every token's KV row and index key, through the library's store/quantise
        slots = np.concatenate([pt[b, np.arange(L) // DSA_PAGE].astype(np.int64) * DSA_PAGE +
                                np.arange(L) % DSA_PAGE for b, L in enumerate(w.seq_lens)])
        slots_t = i32(slots)
        csa.csa_kv_store(data["kv"].contiguous(), slots_t, self.kv_fmt, self.kv_cache,
                         status=self.status)
        csa.csa_index_quant(data["idx_k"].contiguous(), self.idx_fmt, self.k_codes, self.k_bsc,
                            self.k_scales, row_map=slots_t, status=self.status)
        # this step's tokens: the last q_lens[b] of each request
        l_off = np.concatenate([[0], np.cumsum(w.seq_lens)])
        new = np.concatenate([np.arange(l_off[b + 1] - q, l_off[b + 1])
                              for b, q in enumerate(w.q_lens)])
        new_t = torch.as_tensor(new, device=data["kv"].device)
        self.new_kv = data["kv"][new_t].contiguous()
        self.new_k = data["idx_k"][new_t].contiguous()
        self.new_slots = i32(slots[new])
        self.q_idx = data["q_idx"].contiguous()
        self.w_head = data["w"].contiguous()
        self.q = data["q"].contiguous()
        nq = w.num_q
        self.q_codes = torch.empty((nq * Hi, cb), dtype=torch.uint8, device=dev)
        self.q_bsc = (torch.empty((nq * Hi, Di // 16), dtype=torch.uint8, device=dev)
                      if w.idx_fmt == "fp4" else None)
        self.q_scales = torch.empty(nq * Hi, dtype=torch.float32, device=dev)
        self.w_fold = torch.empty((nq, Hi), dtype=torch.float32, device=dev)
        self.logit_stride = max(16, (self.max_len + 15) // 16 * 16)
        self.logits = torch.empty((nq, self.logit_stride), dtype=torch.float32, device=dev)
        self.indices = torch.empty((nq, csa.TOPK), dtype=torch.int32, device=dev)
        self.raw_indices = torch.empty((nq, csa.TOPK), dtype=torch.int32, device=dev)
        self.topk_ws = torch.empty(max(1, csa.csa_topk512_workspace_size(nq, self.max_len)),
                                   dtype=torch.uint8, device=dev)
        self.decode = bool((w.q_lens <= 8).all())
        self.attn_ws = torch.empty(
            max(1, csa.csa_sparse_mqa_workspace_size(nq, w.heads, w.window, self.decode)),
            dtype=torch.uint8, device=dev)
        self.out = torch.empty((nq, w.heads, csa.KV_LATENT), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((nq, w.heads), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        self.check_status()

    def check_status(self):
        s = int(self.status.item())
        if s != 0:
            raise csa.CsaError("device status", s)

    def store(self, stream=None):
        csa.csa_kv_store(self.new_kv, self.new_slots, self.kv_fmt, self.kv_cache,
                         status=self.status, stream=stream)
        csa.csa_index_quant(self.new_k, self.idx_fmt, self.k_codes, self.k_bsc, self.k_scales,
                            row_map=self.new_slots, status=self.status, stream=stream)

    def index(self, stream=None):
        w = self.w
        csa.csa_index_quant(self.q_idx, self.idx_fmt, self.q_codes, self.q_bsc, self.q_scales,
                            w_in=self.w_head, w_out=self.w_fold, status=self.status,
                            stream=stream)
        csa.csa_dsa_indexer_logits(self.q_codes, self.q_bsc, self.w_fold, w.idx_heads, w.idx_dim,
                                   self.idx_fmt, self.k_codes, self.k_bsc, self.k_scales,
                                   self.page_table, self.seq_lens, self.cu_q, self.q_pos,
                                   self.max_len, self.logits, status=self.status, stream=stream)

    def select(self, stream=None):
        csa.csa_dsa_topk512_page_transform(self.logits, self.seq_lens, self.cu_q, self.q_pos,
                                           self.page_table, self.slots_n, self.max_len,
                                           self.indices, self.raw_indices, self.topk_ws,
                                           status=self.status, stream=stream)

    def attend(self, stream=None):
        fn = csa.csa_sparse_mqa_decode if self.decode else csa.csa_sparse_mqa_prefill
        fn(self.q, self.kv_cache, self.kv_cache, self.kv_fmt, self.indices, self.page_table,
           self.seq_lens, self.cu_q, self.q_pos, 0, self.sm_scale, self.out, self.lse,
           self.attn_ws, status=self.status, stream=stream)

    def step(self, stream=None):
        self.store(stream)
        self.index(stream)
        self.select(stream)
        self.attend(stream)
        return self.out
