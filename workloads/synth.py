"""Seeded synthetic decode workloads in the library's cache layouts.

Layouts (all row-major):

* q          bf16  [B][Hq][d]           query head j belongs to KV head j // G
* P          fp32  [Hkv][r][d]          per-KV-head basis with orthonormal rows
* kproj      u8 (FP8 E4M3 codes) or fp32, paged: [num_pages][Hkv][page_size][r]
* kproj_scale fp32 [Hkv]                dequantisation scale per KV head (1 for fp32)
* k_pool, v_pool bf16, paged: [num_pages][page_size][Hkv][d] -- by default views into one pool
                 kv [num_pages][page_size][Hkv][2][d] that holds K then V of each row
* page_table int32 [B][max_pages]       page id of each logical page, -1 where unused
* seq_lens   int32 [B]

Small tensors (queries, bases, page tables, planted positions, gate logits,
linear-branch state) are drawn on the CPU from ``seed`` so that they are the
same whichever device the caches live on; the two large pools are drawn on the
target device.  The projected-key cache is the input the indexer reads: it is
defined as P_h . k for every cached key, quantised to E4M3 with one scale per
KV head (scale = amax / 448) -- that is how the input is specified, not a step
of the decode path.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import torch

FP8_E4M3_MAX = 448.0


@dataclass
class LinearBranchInputs:
    """Caller-owned state of the linear-attention branch, one per (b, KV head)."""

    S: torch.Tensor  # fp32 [B][Hkv][d][d]
    z: torch.Tensor  # fp32 [B][Hkv][d]
    k_new: torch.Tensor  # bf16 [B][Hkv][d]  key of the token being decoded
    v_new: torch.Tensor  # bf16 [B][Hkv][d]
    gate: torch.Tensor  # fp32 [Hq]          gate logit per query head

    def to(self, device) -> "LinearBranchInputs":
        return LinearBranchInputs(*(t.to(device) for t in (self.S, self.z, self.k_new, self.v_new, self.gate)))

    def clone(self) -> "LinearBranchInputs":
        return LinearBranchInputs(*(t.clone() for t in (self.S, self.z, self.k_new, self.v_new, self.gate)))


@dataclass
class DecodeProblem:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    r: int
    M: int
    page_size: int
    num_pages: int
    max_pages: int
    max_seq_len: int
    seq_lens: torch.Tensor
    page_table: torch.Tensor
    q: torch.Tensor
    P: torch.Tensor
    kproj: Optional[torch.Tensor]
    kproj_fp8: bool
    kproj_scale: torch.Tensor
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    softmax_scale: float = 0.0  # 0 means 1/sqrt(d)
    planted: Optional[list] = None  # planted[b][h] -> LongTensor of positions
    lin: Optional[LinearBranchInputs] = None
    kv: Optional[torch.Tensor] = None  # interleaved K|V pool backing k_pool / v_pool, if any
    meta: dict = field(default_factory=dict)

    @property
    def kv_row_stride(self) -> int:
        """Elements between consecutive (page, slot, KV head) rows of the K/V pools (0: separate pools)."""
        return 2 * self.d if self.kv is not None else 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def device(self) -> torch.device:
        return self.k_pool.device

    def to(self, device) -> "DecodeProblem":
        mv = lambda t: None if t is None else t.to(device)
        kv = mv(self.kv)
        return replace(
            self,
            seq_lens=mv(self.seq_lens),
            page_table=mv(self.page_table),
            q=mv(self.q),
            P=mv(self.P),
            kproj=mv(self.kproj),
            kproj_scale=mv(self.kproj_scale),
            k_pool=kv[:, :, :, 0] if kv is not None else mv(self.k_pool),
            v_pool=kv[:, :, :, 1] if kv is not None else mv(self.v_pool),
            kv=kv,
            lin=None if self.lin is None else self.lin.to(device),
        )

    def required_bytes_per_query(self) -> list:
        """Bytes the path must move per sequence: n*r*bytes(kproj) + M_eff*2*d*2 per KV head."""
        eb = 1 if self.kproj_fp8 else 4
        out = []
        for n in self.seq_lens.tolist():
            m_eff = min(self.M, n)
            out.append(self.Hkv * (n * self.r * eb + m_eff * 2 * self.d * 2))
        return out


@dataclass
class LayeredProblem:
    """Several decode layers sharing one page table; indices computed on full layers only."""

    layers: list
    full_layers: tuple

    def source_layer(self, layer: int) -> int:
        return max(f for f in self.full_layers if f <= layer)


def _gen(seed: int, stream: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream * 7919) % (2**63 - 1))
    return g


def _page_layout(seq_lens: Sequence[int], ps: int, paged: bool, gen: torch.Generator, pool_pages=None):
    B = len(seq_lens)
    pages_per_seq = [max(1, -(-n // ps)) for n in seq_lens]
    max_pages = max(pages_per_seq)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    if not paged:
        num_pages = B * max_pages
        for b, npg in enumerate(pages_per_seq):
            table[b, :npg] = torch.arange(b * max_pages, b * max_pages + npg, dtype=torch.int32)
    else:
        total = sum(pages_per_seq)
        num_pages = pool_pages if pool_pages is not None else total
        assert num_pages >= total
        perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
        off = 0
        for b, npg in enumerate(pages_per_seq):
            table[b, :npg] = perm[off : off + npg]
            off += npg
    return table, num_pages, max_pages


def _orthonormal_basis(Hkv: int, r: int, d: int, gen: torch.Generator, bf16_values: bool) -> torch.Tensor:
    """r x d bases with orthonormal rows: QR of a seeded Gaussian d x r matrix, transposed."""
    P = torch.empty(Hkv, r, d, dtype=torch.float64)
    for h in range(Hkv):
        A = torch.randn(d, r, generator=gen, dtype=torch.float64)
        Qm, _ = torch.linalg.qr(A)
        P[h] = Qm.T
    P32 = P.to(torch.float32)
    if bf16_values:
        P32 = P32.to(torch.bfloat16).to(torch.float32)
    return P32


def _project_pool(k_pool: torch.Tensor, P: torch.Tensor, fp8: bool):
    """Projected-key cache for every pool row (input definition), quantised per KV head."""
    num_pages, ps, Hkv, d = k_pool.shape
    r = P.shape[1]
    dev = k_pool.device
    Pd = P.to(dev)
    proj = torch.empty(num_pages, Hkv, ps, r, dtype=torch.float32, device=dev)
    chunk = max(1, (1 << 23) // (ps * Hkv * d))
    for p0 in range(0, num_pages, chunk):
        kf = k_pool[p0 : p0 + chunk].to(torch.float32)
        proj[p0 : p0 + chunk] = torch.einsum("cshd,hrd->chsr", kf, Pd)
    if not fp8:
        return proj, torch.ones(Hkv, dtype=torch.float32)
    amax = proj.abs().amax(dim=(0, 2, 3)).to(torch.float32)
    scale = torch.where(amax > 0, amax / FP8_E4M3_MAX, torch.ones_like(amax))
    codes = torch.empty(num_pages, Hkv, ps, r, dtype=torch.uint8, device=dev)
    inv = (1.0 / scale).view(1, Hkv, 1, 1)
    for p0 in range(0, num_pages, chunk):
        x = (proj[p0 : p0 + chunk] * inv).clamp_(-FP8_E4M3_MAX, FP8_E4M3_MAX)
        codes[p0 : p0 + chunk] = x.to(torch.float8_e4m3fn).view(torch.uint8)
    del proj
    return codes, scale.cpu()


def _rows_of(table: torch.Tensor, ps: int, b: int, pos: torch.Tensor):
    pages = table[b, (pos // ps)].long()
    slots = (pos % ps).long()
    return pages, slots


def make_problem(
    *,
    name: str,
    B: int,
    Hq: int,
    Hkv: int,
    d: int,
    r: int,
    M: int,
    seq_lens: Sequence[int],
    page_size: int = 64,
    paged: bool = False,
    pool_pages: Optional[int] = None,
    kproj_fp8: bool = True,
    plant: tuple = ("none",),
    seed: int = 0,
    device="cpu",
    bf16_basis: bool = False,
    linear: bool = False,
    softmax_scale: float = 0.0,
    with_kproj: bool = True,
    kv_interleaved: bool = True,
) -> DecodeProblem:
    """Draw one decode problem.

    plant: ("none",) | ("shifted", count) -> k = 2*qdir_mean + N(0, 0.1^2)
           | ("cosine", frac) -> k = sqrt(d)*(0.5*qhat + sqrt(3)/2*w), w unit, w ⟂ qhat
    """
    assert Hq % Hkv == 0
    device = torch.device(device)
    seq_lens = [int(n) for n in seq_lens]
    assert len(seq_lens) == B and min(seq_lens) >= 1
    G = Hq // Hkv
    g_layout = _gen(seed, 1)
    table, num_pages, max_pages = _page_layout(seq_lens, page_size, paged, g_layout, pool_pages)
    g_small = _gen(seed, 2)
    q = torch.randn(B, Hq, d, generator=g_small).to(torch.bfloat16)
    P = _orthonormal_basis(Hkv, r, d, _gen(seed, 3), bf16_basis)

    g_dev = _gen(seed, 4, device)
    kv = None
    if kv_interleaved:
        kv = torch.randn(num_pages, page_size, Hkv, 2, d, generator=g_dev, device=device, dtype=torch.bfloat16)
        k_pool, v_pool = kv[:, :, :, 0], kv[:, :, :, 1]
    else:
        k_pool = torch.randn(num_pages, page_size, Hkv, d, generator=g_dev, device=device, dtype=torch.bfloat16)
        v_pool = torch.randn(num_pages, page_size, Hkv, d, generator=g_dev, device=device, dtype=torch.bfloat16)

    planted = None
    if plant[0] != "none":
        g_pl = _gen(seed, 5)
        planted = []
        qf = q.to(torch.float32)
        for b in range(B):
            n = seq_lens[b]
            row = []
            for h in range(Hkv):
                qsum = qf[b, h * G : (h + 1) * G].sum(0)  # direction of the group's queries
                if plant[0] == "shifted":
                    cnt = min(int(plant[1]), n)
                    pos = torch.randperm(n, generator=g_pl)[:cnt]
                    vec = 2.0 * (qsum / G) + 0.1 * torch.randn(cnt, d, generator=g_pl)
                elif plant[0] == "cosine":
                    cnt = min(n, max(1, int(round(float(plant[1]) * n))))
                    pos = torch.randperm(n, generator=g_pl)[:cnt]
                    qhat = qsum / qsum.norm()
                    w = torch.randn(cnt, d, generator=g_pl)
                    w = w - (w @ qhat)[:, None] * qhat[None, :]
                    w = w / w.norm(dim=1, keepdim=True)
                    vec = math.sqrt(d) * (0.5 * qhat[None, :] + (math.sqrt(3.0) / 2.0) * w)
                else:
                    raise ValueError(plant)
                pages, slots = _rows_of(table, page_size, b, pos)
                k_pool[pages.to(device), slots.to(device), h] = vec.to(torch.bfloat16).to(device)
                row.append(pos.sort().values)
            planted.append(row)

    if with_kproj:
        kproj, kscale = _project_pool(k_pool, P, kproj_fp8)
    else:
        kproj, kscale = None, torch.ones(Hkv, dtype=torch.float32)

    lin = None
    if linear:
        g_lin = _gen(seed, 6)
        # Caller-owned state standing for a prefix of n-1 tokens: entries of the
        # magnitude such a prefix gives (S ~ sqrt(n-1), z ~ n-1, z > 0).
        nm1 = torch.tensor([max(1, n - 1) for n in seq_lens], dtype=torch.float32)
        S = torch.randn(B, Hkv, d, d, generator=g_lin) * nm1.sqrt().view(B, 1, 1, 1)
        z = (1.0 + 0.5 * torch.rand(B, Hkv, d, generator=g_lin)) * nm1.view(B, 1, 1)
        gate = torch.randn(Hq, generator=g_lin).to(torch.bfloat16).to(torch.float32)
        k_new = torch.empty(B, Hkv, d, dtype=torch.bfloat16)
        v_new = torch.empty(B, Hkv, d, dtype=torch.bfloat16)
        for b in range(B):
            last = torch.tensor([seq_lens[b] - 1])
            pages, slots = _rows_of(table, page_size, b, last)
            k_new[b] = k_pool[pages.to(device), slots.to(device)][0].cpu()
            v_new[b] = v_pool[pages.to(device), slots.to(device)][0].cpu()
        lin = LinearBranchInputs(S, z, k_new, v_new, gate)

    prob = DecodeProblem(
        name=name,
        B=B,
        Hq=Hq,
        Hkv=Hkv,
        d=d,
        r=r,
        M=M,
        page_size=page_size,
        num_pages=num_pages,
        max_pages=max_pages,
        max_seq_len=max(seq_lens),
        seq_lens=torch.tensor(seq_lens, dtype=torch.int32),
        page_table=table,
        q=q,
        P=P,
        kproj=kproj,
        kproj_fp8=kproj_fp8,
        kproj_scale=kscale,
        k_pool=k_pool,
        v_pool=v_pool,
        softmax_scale=softmax_scale,
        planted=planted,
        lin=lin,
        kv=kv,
        meta={"seed": seed, "paged": paged, "plant": plant},
    )
    return prob.to(device)


# ---------------------------------------------------------------------------
# The five workloads.  Each accepts size overrides so that tests can draw the
# same structure at sizes the oracle finishes in seconds.
# ---------------------------------------------------------------------------

CONFIG_NAMES = {
    1: "tiny decode: B=1, 4q/1kv, d=64, n=1024, r=16, M=64, fp32 projected keys",
    2: "GQA decode 16K: B=8, 32q/8kv, d=128, n=16384, r=32, M=2048, FP8 projected keys, contiguous",
    3: "long-context decode 128K: B=16, 64q/8kv, d=128, n=131072, r=32, M=2048, paged ps=64, FP8",
    4: "ragged paged batch: 64 seqs, n~U[4096,131072], 32q/8kv, d=128, r=32, M=min(2048,n), FP8",
    5: "hybrid: 8 layers, B=8, 32q/8kv, d=128, n=32768, r=32, M=1024, linear branch + gate, reuse from layers 0,4",
}


def config1(device="cpu", seed=1001, **kw) -> DecodeProblem:
    args = dict(B=1, Hq=4, Hkv=1, d=64, r=16, M=64, n=1024)
    args.update(kw)
    n = args.pop("n")
    return make_problem(
        name="config1", seq_lens=[n] * args["B"], page_size=64, paged=False, kproj_fp8=False,
        plant=("shifted", 8), seed=seed, device=device, **args,
    )


def config2(device="cpu", seed=1002, **kw) -> DecodeProblem:
    args = dict(B=8, Hq=32, Hkv=8, d=128, r=32, M=2048, n=16384)
    args.update(kw)
    n = args.pop("n")
    return make_problem(
        name="config2", seq_lens=[n] * args["B"], page_size=64, paged=False, kproj_fp8=True,
        plant=("cosine", 0.01), seed=seed, device=device, **args,
    )


def config3(device="cpu", seed=1003, **kw) -> DecodeProblem:
    args = dict(B=16, Hq=64, Hkv=8, d=128, r=32, M=2048, n=131072, paged=True)
    args.update(kw)
    n = args.pop("n")
    return make_problem(
        name="config3", seq_lens=[n] * args["B"], page_size=64, kproj_fp8=True,
        plant=("cosine", 0.005), seed=seed, device=device, **args,
    )


def config4(device="cpu", seed=1004, num_seqs=64, n_lo=4096, n_hi=131072, **kw) -> DecodeProblem:
    args = dict(Hq=32, Hkv=8, d=128, r=32, M=2048)
    args.update(kw)
    g = _gen(seed, 9)
    lens = torch.randint(n_lo, n_hi + 1, (num_seqs,), generator=g).tolist()
    return make_problem(
        name="config4", B=num_seqs, seq_lens=lens, page_size=64, paged=True, kproj_fp8=True,
        plant=("none",), seed=seed, device=device, **args,
    )


def config5(device="cpu", seed=1005, layers=8, full_layers=(0, 4), **kw) -> LayeredProblem:
    args = dict(B=8, Hq=32, Hkv=8, d=128, r=32, M=1024, n=32768)
    args.update(kw)
    n = args.pop("n")
    out = []
    for layer in range(layers):
        out.append(
            make_problem(
                name=f"config5.layer{layer}", seq_lens=[n] * args["B"], page_size=64, paged=False,
                kproj_fp8=True, plant=("cosine", 0.01), seed=seed * 100 + layer, device=device,
                bf16_basis=True, linear=True, with_kproj=(layer in full_layers), **args,
            )
        )
    return LayeredProblem(layers=out, full_layers=tuple(full_layers))
