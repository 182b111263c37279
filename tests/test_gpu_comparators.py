"""The comparators the pages measure against, built from the library's own kernels: full attention
over every cached position (lisa_dense_decode_attn) and "gather, then attend" (lisa_gather_kv into a
contiguous buffer, then dense attention over it).  Both are checked against the oracle."""

import ctypes

import numpy as np
import pytest
import torch

import indexed_top_sparse_b200 as L
from indexed_top_sparse_b200 import binding as Bnd
from oracle import lisa_oracle as O
from tests.parity import check_outputs
from workloads import make_problem
from workloads import run as R
from workloads.host_view import host_inputs


def f64(t):
    return t.detach().float().cpu().double().numpy()


DENSE_CASES = {
    "paged_g8_d128": dict(B=2, Hq=16, Hkv=2, d=128, r=32, M=64, seq_lens=[3000, 777], page_size=64, paged=True),
    "contig_g4_d64": dict(B=3, Hq=8, Hkv=2, d=64, r=16, M=64, seq_lens=[1024, 1, 65], page_size=16, paged=False),
    "g1_page1024": dict(B=1, Hq=2, Hkv=2, d=128, r=32, M=64, seq_lens=[5000], page_size=1024, paged=True),
    "separate_pools": dict(B=2, Hq=4, Hkv=1, d=128, r=32, M=64, seq_lens=[2100, 300], page_size=64, paged=True,
                           kv_interleaved=False),
}


@pytest.mark.gpu
@pytest.mark.parametrize("case", list(DENSE_CASES))
def test_dense_attention_matches_oracle(cuda_device, case):
    prob = make_problem(name=case, device=cuda_device, kproj_fp8=True, plant=("none",), seed=500 + len(case),
                        **DENSE_CASES[case])
    out, lse, ws = R.dense_attention(prob)
    assert L.lisa_check_device_error(ws) == 0
    inp = host_inputs(prob)
    inp["M"] = int(max(prob.seq_lens.tolist()))  # every position selected: full attention
    ref = O.decode_step(inp)
    pairs = [(b, h) for b in range(prob.B) for h in range(prob.Hkv)]
    check_outputs(f64(out), ref["out"], pairs, prob.G)
    assert np.allclose(lse.cpu().numpy(), ref["lse"], rtol=1e-4, atol=1e-4)


@pytest.mark.gpu
def test_gather_then_attend_matches_in_place_attention(cuda_device):
    prob = make_problem(name="gta", device=cuda_device, B=3, Hq=16, Hkv=2, d=128, r=32, M=256,
                        seq_lens=[6000, 200, 3000], page_size=64, paged=True, kproj_fp8=True, plant=("cosine", 0.01),
                        seed=520)
    ws = R.workspace(prob)
    idx, count = R.index_topm(prob, ws)
    direct, _ = R.attention(prob, idx, count, ws)
    gta = R.GatherThenAttend(prob, count)
    gta.gather(idx)
    out, _ = gta.attend()
    assert L.lisa_check_device_error(gta.ws_gather) == 0 and L.lisa_check_device_error(gta.ws_attn) == 0
    # the gathered rows are the pool rows, bit for bit, and zeros past the count
    inp = host_inputs(prob)
    g = gta.gathered.view(prob.B, prob.Hkv, prob.M, 2, prob.d).cpu().view(torch.int16).numpy().view(np.uint16)
    for b in range(prob.B):
        for h in range(prob.Hkv):
            n = int(count[b, h])
            for i in list(range(min(n, 5))) + [n - 1]:
                t = int(idx[b, h, i])
                pg, s = inp["page_table"][b][t // prob.page_size], t % prob.page_size
                assert np.array_equal(g[b, h, i, 0], inp["k_pool"][pg, s, h])
                assert np.array_equal(g[b, h, i, 1], inp["v_pool"][pg, s, h])
            assert not g[b, h, n:].any()
    # both attentions equal the oracle's attention over the GPU's index sets
    sets = [[idx[b, h, : int(count[b, h])].cpu().numpy() for h in range(prob.Hkv)] for b in range(prob.B)]
    ref = O.decode_step(inp, reuse_idx=sets)
    pairs = [(b, h) for b in range(prob.B) for h in range(prob.Hkv)]
    check_outputs(f64(direct), ref["out"], pairs, prob.G)
    check_outputs(f64(out), ref["out"], pairs, prob.G)


def test_dense_rejects_contexts_beyond_the_merge():
    # one sequence of 262,144 positions needs more than 256 partials per (b, KV head)
    d = L.make_desc(batch=1, num_q_heads=8, num_kv_heads=1, head_dim=128, idx_dim=32, budget_m=2048, page_size=1024,
                    max_pages_per_seq=256, max_seq_len=262144, num_pages=256)
    d.seq_lens = 0x1000
    d.page_table = 0x2000
    A = 0x1000
    st = Bnd._lib.lisa_dense_decode_attn(ctypes.byref(d), A, A, A, A, None, A, 1 << 30, None)
    assert st == 2  # LISA_ERR_UNSUPPORTED, before anything touches the GPU
