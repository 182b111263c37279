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
