"""Host (numpy) copies of a DecodeProblem in the same layouts, for CPU checkers.

Only dtype/device plumbing: bf16 tensors become their uint16 bit patterns,
FP8 caches their uint8 codes.  For large problems a subset of sequences can be
extracted; their pages are copied into a compact pool and the page table is
renumbered, so the consumer still reads through a page table.
"""

from __future__ import annotations

from typing import Optional, Sequence

import numpy as np
import torch

from .synth import DecodeProblem


def _bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def host_inputs(prob: DecodeProblem, seqs: Optional[Sequence[int]] = None, lin=None) -> dict:
    """numpy view of prob (optionally only the sequences in seqs, renumbered 0..len-1)."""
    ps = prob.page_size
    seqs = list(range(prob.B)) if seqs is None else [int(s) for s in seqs]
    table = prob.page_table.cpu()
    lens = prob.seq_lens.cpu()
    sub_lens = lens[seqs]
    pages_needed = [(-(-int(n) // ps)) for n in sub_lens.tolist()]
    max_pages = max(pages_needed)
    src_pages = []
    new_table = np.full((len(seqs), max_pages), -1, dtype=np.int64)
    for i, b in enumerate(seqs):
        npg = pages_needed[i]
        new_table[i, :npg] = np.arange(len(src_pages), len(src_pages) + npg)
        src_pages.extend(table[b, :npg].tolist())
    src = torch.tensor(src_pages, dtype=torch.long, device=prob.k_pool.device)
    out = {
        "B": len(seqs),
        "Hq": prob.Hq,
        "Hkv": prob.Hkv,
        "d": prob.d,
        "r": prob.r,
        "M": prob.M,
        "page_size": ps,
        "softmax_scale": float(prob.softmax_scale),
        "seq_lens": sub_lens.numpy().astype(np.int64),
        "page_table": new_table,
        "q": _bits16(prob.q[torch.tensor(seqs, device=prob.q.device)]),
        "P": prob.P.cpu().numpy().astype(np.float64),
        "kproj_fp8": bool(prob.kproj_fp8),
        "kproj_scale": prob.kproj_scale.cpu().numpy().astype(np.float64),
        "k_pool": _bits16(prob.k_pool.index_select(0, src)),
        "v_pool": _bits16(prob.v_pool.index_select(0, src)),
    }
    if prob.kproj is not None:
        kp = prob.kproj.index_select(0, src).cpu()
        out["kproj"] = kp.numpy() if prob.kproj_fp8 else kp.numpy().astype(np.float64)
    lin = prob.lin if lin is None else lin
    if lin is not None:
        sel = torch.tensor(seqs, device=lin.S.device)
        out["lin"] = {
            "S": lin.S[sel].cpu().numpy().astype(np.float64),
            "z": lin.z[sel].cpu().numpy().astype(np.float64),
            "k_new": _bits16(lin.k_new[sel]),
            "v_new": _bits16(lin.v_new[sel]),
            "gate": lin.gate.cpu().numpy().astype(np.float64),
        }
    return out
