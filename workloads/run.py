"""Drive the library's C entry points on a DecodeProblem (device tensors in, device tensors out).

Marshalling only: descriptors, output buffers and workspace come from here;
every step of the decode path runs inside the library.
"""

from __future__ import annotations

from typing import Optional

import torch

import indexed_top_sparse_b200 as L

from .synth import DecodeProblem


def desc_of(prob: DecodeProblem) -> L.DecodeDesc:
    return L.make_desc(
        batch=prob.B, num_q_heads=prob.Hq, num_kv_heads=prob.Hkv, head_dim=prob.d, idx_dim=prob.r,
        budget_m=prob.M, page_size=prob.page_size, max_pages_per_seq=prob.max_pages,
        max_seq_len=prob.max_seq_len, num_pages=prob.num_pages, seq_lens=prob.seq_lens,
        page_table=prob.page_table, softmax_scale=prob.softmax_scale, kv_row_stride=prob.kv_row_stride,
    )


def kv_args(prob: DecodeProblem):
    """(k_pool, v_pool) arguments of the library: the interleaved pool and its V half, or the two pools."""
    if prob.kv is not None:
        return prob.kv, L.DevicePtr(prob.kv.data_ptr() + prob.d * prob.kv.element_size())
    return prob.k_pool, prob.v_pool


def kproj_dtype(prob: DecodeProblem) -> int:
    return L.KPROJ_FP8_E4M3 if prob.kproj_fp8 else L.KPROJ_FP32


def workspace(prob: DecodeProblem, desc=None) -> torch.Tensor:
    return L.alloc_workspace(desc or desc_of(prob), prob.device)


def index_scores(prob: DecodeProblem, ws: torch.Tensor, desc=None) -> torch.Tensor:
    desc = desc or desc_of(prob)
    scores = torch.full((prob.B, prob.Hkv, prob.max_seq_len), float("nan"), dtype=torch.float32, device=prob.device)
    L.lisa_index_score(desc, prob.q, prob.P, prob.kproj, kproj_dtype(prob), prob.kproj_scale.to(prob.device), scores, ws)
    return scores


def topm_from_scores(prob: DecodeProblem, scores: torch.Tensor, ws: torch.Tensor, desc=None):
    desc = desc or desc_of(prob)
    idx = torch.full((prob.B, prob.Hkv, prob.M), -7, dtype=torch.int32, device=prob.device)
    count = torch.full((prob.B, prob.Hkv), -7, dtype=torch.int32, device=prob.device)
    L.lisa_topm_select(desc, scores, idx, count, ws)
    return idx, count


def index_topm(prob: DecodeProblem, ws: torch.Tensor, desc=None):
    desc = desc or desc_of(prob)
    idx = torch.full((prob.B, prob.Hkv, prob.M), -7, dtype=torch.int32, device=prob.device)
    count = torch.full((prob.B, prob.Hkv), -7, dtype=torch.int32, device=prob.device)
    L.lisa_index_topm(desc, prob.q, prob.P, prob.kproj, kproj_dtype(prob), prob.kproj_scale.to(prob.device), idx,
                      count, ws)
    return idx, count


def attention(prob: DecodeProblem, idx: torch.Tensor, count: torch.Tensor, ws: torch.Tensor, desc=None):
    desc = desc or desc_of(prob)
    out = torch.empty(prob.B, prob.Hq, prob.d, dtype=torch.bfloat16, device=prob.device)
    lse = torch.empty(prob.B, prob.Hq, dtype=torch.float32, device=prob.device)
    k, v = kv_args(prob)
    L.lisa_sparse_decode_attn(desc, prob.q, k, v, idx, count, out, lse, ws)
    return out, lse


def fused(prob: DecodeProblem, ws: torch.Tensor, desc=None, reuse: Optional[tuple] = None, return_idx=True,
          lin=None, events=None, stream=None, out=None, lse=None):
    """One call of lisa_fused_decode.  lin: a workloads LinearBranchInputs (state updated in place)."""
    desc = desc or desc_of(prob)
    dev = prob.device
    out = out if out is not None else torch.empty(prob.B, prob.Hq, prob.d, dtype=torch.bfloat16, device=dev)
    lse = lse if lse is not None else torch.empty(prob.B, prob.Hq, dtype=torch.float32, device=dev)
    idx = count = None
    if return_idx and reuse is None:
        idx = torch.full((prob.B, prob.Hkv, prob.M), -7, dtype=torch.int32, device=dev)
        count = torch.full((prob.B, prob.Hkv), -7, dtype=torch.int32, device=dev)
    lb = None
    if lin is not None:
        lb = L.linear_branch(lin.S, lin.z, lin.k_new, lin.v_new, lin.gate)
    ridx, rcount = (None, None) if reuse is None else reuse
    scale = prob.kproj_scale.to(dev) if prob.kproj is not None else None
    k, v = kv_args(prob)
    L.lisa_fused_decode(desc, prob.q, prob.P, prob.kproj, kproj_dtype(prob), scale, k, v, ridx,
                        rcount, idx, count, lb, out, lse, ws, events=events, stream=stream)
    return {"out": out, "lse": lse, "idx": idx, "count": count}


# ---- comparators (not on the decode path) ----

def dense_attention(prob: DecodeProblem, desc=None):
    """lisa_dense_decode_attn: every query head over all n_b positions."""
    desc = desc or desc_of(prob)
    ws = L.alloc_dense_workspace(desc, prob.device)
    out = torch.empty(prob.B, prob.Hq, prob.d, dtype=torch.bfloat16, device=prob.device)
    lse = torch.empty(prob.B, prob.Hq, dtype=torch.float32, device=prob.device)
    k, v = kv_args(prob)
    L.lisa_dense_decode_attn(desc, prob.q, k, v, out, lse, ws)
    return out, lse, ws


class GatherThenAttend:
    """The "gather, then attend" baseline: lisa_gather_kv into a contiguous [B*Hkv][M][2][d] buffer,
    then lisa_dense_decode_attn over it as B*Hkv sequences of one KV head (identity page table)."""

    def __init__(self, prob: DecodeProblem, count: torch.Tensor):
        if prob.M % 64 != 0:
            raise ValueError("the gathered buffer is paged in 64-row pages: M must be a multiple of 64")
        dev = prob.device
        self.prob = prob
        self.Bp, self.pages = prob.B * prob.Hkv, prob.M // 64
        self.gathered = torch.empty(self.Bp, prob.M, 2, prob.d, dtype=torch.bfloat16, device=dev)
        self.table = torch.arange(self.Bp * self.pages, dtype=torch.int32, device=dev).view(self.Bp, self.pages)
        self.count = count
        self.desc = L.make_desc(batch=self.Bp, num_q_heads=prob.G, num_kv_heads=1, head_dim=prob.d, idx_dim=prob.r,
                                budget_m=prob.M, page_size=64, max_pages_per_seq=self.pages, max_seq_len=prob.M,
                                num_pages=self.Bp * self.pages, seq_lens=count.view(-1), page_table=self.table,
                                softmax_scale=prob.softmax_scale, kv_row_stride=2 * prob.d)
        self.ws_gather = L.alloc_workspace(desc_of(prob), dev)
        self.ws_attn = L.alloc_dense_workspace(self.desc, dev)
        self.out = torch.empty(prob.B, prob.Hq, prob.d, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(prob.B, prob.Hq, dtype=torch.float32, device=dev)

    def gather(self, idx: torch.Tensor, stream=None):
        k, v = kv_args(self.prob)
        L.lisa_gather_kv(desc_of(self.prob), idx, self.count, k, v, self.gathered, self.ws_gather, stream=stream)

    def attend(self, stream=None):
        v = L.DevicePtr(self.gathered.data_ptr() + self.prob.d * 2)
        L.lisa_dense_decode_attn(self.desc, self.prob.q, self.gathered, v, self.out, self.lse, self.ws_attn,
                                 stream=stream)
        return self.out, self.lse
