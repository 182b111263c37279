"""GPU parity of lisa_index_score_multi (T query tokens per sequence on the tensor cores) with the
oracle, and of the per-token top-M that lisa_topm_select computes from its scores."""

import numpy as np
import pytest
import torch

import indexed_top_sparse_b200 as L
from oracle import lisa_oracle as O
from workloads import make_problem
from workloads import run as R
from workloads.host_view import host_inputs

pytestmark = pytest.mark.gpu


def _bits16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("T,r,d,page", [(4, 32, 128, 64), (8, 32, 128, 16), (1, 16, 64, 64), (3, 16, 128, 1024),
                                          (6, 32, 128, 256), (2, 16, 128, 32), (5, 16, 64, 128)])
def test_multi_query_scores_and_selection(cuda_device, T, r, d, page):
    prob = make_problem(name="mq", device=cuda_device, B=2, Hq=8, Hkv=2, d=d, r=r, M=128,
                        seq_lens=[6000, 700], page_size=page, paged=True, kproj_fp8=True, plant=("cosine", 0.01),
                        seed=600 + T)
    g = torch.Generator().manual_seed(601 + T)
    qt = torch.randn(prob.B, T, prob.Hq, prob.d, generator=g).to(torch.bfloat16).to(cuda_device)
    desc = R.desc_of(prob)
    ws = R.workspace(prob, desc)
    scores = torch.full((prob.B, T, prob.Hkv, prob.max_seq_len), float("nan"), dtype=torch.float32,
                        device=cuda_device)
    L.lisa_index_score_multi(desc, T, qt, prob.P, prob.kproj, L.KPROJ_FP8_E4M3, prob.kproj_scale.to(cuda_device),
                             scores, ws)
    assert L.lisa_check_device_error(ws) == 0
    inp = host_inputs(prob)
    qb = _bits16(qt)
    got = scores.cpu().double().numpy()
    lens = inp["seq_lens"]
    for b in range(prob.B):
        n = int(lens[b])
        for h in range(prob.Hkv):
            ref = O.multi_query_scores(inp, qb, T, b, h)
            for j in range(T):
                lim = n - T + j + 1
                tol = 1e-5 * np.max(np.abs(ref[j, :lim]))
                assert np.all(np.abs(got[b, j, h, :lim] - ref[j, :lim]) <= tol)
                assert np.all(np.isnan(got[b, j, h, lim:]))  # later positions are not written
    # top-M per token: a desc of B*T sequences (b*T + j) of length n_b - T + j + 1 over the same scores
    lens_bt = torch.tensor([int(lens[b]) - T + j + 1 for b in range(prob.B) for j in range(T)], dtype=torch.int32,
                           device=cuda_device)
    table_bt = prob.page_table.repeat_interleave(T, dim=0).contiguous()
    desc_bt = L.make_desc(batch=prob.B * T, num_q_heads=prob.Hq, num_kv_heads=prob.Hkv, head_dim=prob.d,
                          idx_dim=prob.r, budget_m=prob.M, page_size=prob.page_size,
                          max_pages_per_seq=prob.max_pages, max_seq_len=prob.max_seq_len,
                          num_pages=prob.num_pages, seq_lens=lens_bt, page_table=table_bt)
    ws_bt = L.alloc_workspace(desc_bt, cuda_device)
    idx = torch.full((prob.B * T, prob.Hkv, prob.M), -7, dtype=torch.int32, device=cuda_device)
    cnt = torch.full((prob.B * T, prob.Hkv), -7, dtype=torch.int32, device=cuda_device)
    L.lisa_topm_select(desc_bt, scores.view(prob.B * T, prob.Hkv, prob.max_seq_len), idx, cnt, ws_bt)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(prob.B):
        for j in range(T):
            lim = int(lens[b]) - T + j + 1
            for h in range(prob.Hkv):
                want = O.select_top_m(got[b, j, h, :lim], prob.M)  # exact on the GPU's own scores
                k = int(cnt_h[b * T + j, h])
                assert k == len(want) and np.array_equal(idx_h[b * T + j, h, :k], want)


@pytest.mark.parametrize("T,r,d,page,M,lens", [
    (4, 32, 128, 64, 128, [6000, 130, 2]),
    (8, 32, 128, 16, 256, [20000, 700]),
    (3, 16, 64, 1024, 128, [9000, 129]),
    (1, 32, 128, 64, 512, [20000]),
    (6, 16, 128, 128, 64, [5000, 4097]),
])
def test_fused_multi_query_topm(cuda_device, T, r, d, page, M, lens):
    """lisa_index_topm_multi against the oracle's exact per-token sets over its own fp64 scores."""
    from tests.parity import check_index_sets

    B = len(lens)
    prob = make_problem(name="mqt", device=cuda_device, B=B, Hq=8, Hkv=2, d=d, r=r, M=M, seq_lens=lens,
                        page_size=page, paged=True, kproj_fp8=True, plant=("cosine", 0.01), seed=700 + T)
    g = torch.Generator().manual_seed(701 + T)
    qt = torch.randn(B, T, prob.Hq, prob.d, generator=g).to(torch.bfloat16).to(cuda_device)
    desc = R.desc_of(prob)
    ws = L.alloc_workspace_multi(desc, T, cuda_device)
    idx = torch.full((B, T, prob.Hkv, M), -7, dtype=torch.int32, device=cuda_device)
    cnt = torch.full((B, T, prob.Hkv), -7, dtype=torch.int32, device=cuda_device)
    L.lisa_index_topm_multi(desc, T, qt, prob.P, prob.kproj, L.KPROJ_FP8_E4M3, prob.kproj_scale.to(cuda_device),
                            idx, cnt, ws)
    assert L.lisa_check_device_error(ws) == 0
    inp = host_inputs(prob)
    qb = _bits16(qt)
    ref = {"idx": [], "scores": []}
    lims = []
    for b in range(B):
        n = int(inp["seq_lens"][b])
        per_h = [O.multi_query_scores(inp, qb, T, b, h) for h in range(prob.Hkv)]
        for j in range(T):
            lim = max(0, n - T + j + 1)
            lims.append(lim)
            ref["scores"].append([per_h[h][j, :lim] for h in range(prob.Hkv)])
            ref["idx"].append([O.select_top_m(per_h[h][j, :lim], M) for h in range(prob.Hkv)])
    pairs = [(bj, h) for bj in range(B * T) for h in range(prob.Hkv)]
    same = check_index_sets(idx.view(B * T, prob.Hkv, M).cpu().numpy(), cnt.view(B * T, prob.Hkv).cpu().numpy(),
                            ref, lims, M, pairs)
    assert len(same) >= 0.9 * len(pairs)


def test_fused_multi_query_topm_rejects_bad_token_counts(cuda_device):
    prob = make_problem(name="mqt", device=cuda_device, B=1, Hq=8, Hkv=2, d=128, r=32, M=64, seq_lens=[300],
                        page_size=64, paged=True, kproj_fp8=True, seed=5)
    desc = R.desc_of(prob)
    assert L.lisa_workspace_size_multi(desc, 0) == 0 and L.lisa_workspace_size_multi(desc, 9) == 0
    ws = L.alloc_workspace_multi(desc, 2, cuda_device)
    qt = torch.zeros(1, 9, prob.Hq, prob.d, dtype=torch.bfloat16, device=cuda_device)
    idx = torch.empty(1, 9, prob.Hkv, 64, dtype=torch.int32, device=cuda_device)
    cnt = torch.empty(1, 9, prob.Hkv, dtype=torch.int32, device=cuda_device)
    with pytest.raises(L.LisaError):
        L.lisa_index_topm_multi(desc, 9, qt, prob.P, prob.kproj, L.KPROJ_FP8_E4M3, prob.kproj_scale.to(cuda_device),
                                idx, cnt, ws)
    with pytest.raises(L.LisaError):  # the workspace of T = 2 is too small for T = 8
        L.lisa_index_topm_multi(desc, 8, qt, prob.P, prob.kproj, L.KPROJ_FP8_E4M3,
                                prob.kproj_scale.to(cuda_device), idx, cnt, ws)
