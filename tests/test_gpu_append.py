"""GPU parity of lisa_append_token (the producer side of the caches) with the oracle.

The K/V rows, the E4M3 codes and the fp32 projected keys written by the library must equal the
oracle's bit for bit -- the codes are integers decided by the fixed fp32 arithmetic both sides
follow -- and every other byte of the pools must be unchanged.
"""

import numpy as np
import pytest
import torch

import indexed_top_sparse_b200 as L
from oracle import lisa_oracle as O
from workloads import config3, make_problem
from workloads import run as R

pytestmark = pytest.mark.gpu


def _bits16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _new_rows(prob, seed):
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn(prob.B, prob.Hkv, prob.d, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(prob.B, prob.Hkv, prob.d, generator=g).to(torch.bfloat16)
    return k.to(prob.device), v.to(prob.device)


def _pools(prob):
    kp = prob.kproj.cpu().numpy() if prob.kproj_fp8 else prob.kproj.cpu().numpy().astype(np.float32)
    return {"k": _bits16(prob.k_pool), "v": _bits16(prob.v_pool), "kproj": kp}


def _append(prob, k_new, v_new, positions=None):
    desc = R.desc_of(prob)
    ws = R.workspace(prob, desc)
    k_arg, v_arg = R.kv_args(prob)
    L.lisa_append_token(desc, positions, k_new, v_new, prob.P, prob.kproj, R.kproj_dtype(prob),
                        prob.kproj_scale.to(prob.device), k_arg, v_arg, ws)
    return ws


def _check(prob, seed, positions=None):
    k_new, v_new = _new_rows(prob, seed)
    before = _pools(prob)
    ws = _append(prob, k_new, v_new, positions)
    assert L.lisa_check_device_error(ws) == 0
    pos = None if positions is None else positions.cpu().numpy()
    want = O.append_token(before, prob.seq_lens.cpu().numpy(), prob.page_table.cpu().numpy(), _bits16(k_new),
                          _bits16(v_new), prob.P.cpu().numpy(), prob.kproj_scale.cpu().numpy(), prob.kproj_fp8,
                          positions=pos)
    got = _pools(prob)
    for name in ("k", "v", "kproj"):
        assert np.array_equal(got[name].view(np.uint8), want[name].view(np.uint8)), name


APPEND_CASES = {
    "fp8_r32_paged_interleaved": dict(B=3, Hq=8, Hkv=2, d=128, r=32, M=64, seq_lens=[700, 65, 1024], page_size=64,
                                      paged=True, kproj_fp8=True),
    "fp8_r16_d64_separate_pools": dict(B=2, Hq=6, Hkv=3, d=64, r=16, M=32, seq_lens=[100, 17], page_size=16,
                                       paged=True, kproj_fp8=True, kv_interleaved=False),
    "fp32_r32_contiguous": dict(B=2, Hq=4, Hkv=1, d=128, r=32, M=32, seq_lens=[300, 1], page_size=64, paged=False,
                                kproj_fp8=False),
    "fp8_g8_page1024": dict(B=2, Hq=16, Hkv=2, d=128, r=32, M=64, seq_lens=[2500, 1025], page_size=1024,
                            paged=True, kproj_fp8=True),
}


@pytest.mark.parametrize("case", list(APPEND_CASES))
def test_append_bit_exact(cuda_device, case):
    prob = make_problem(name=case, device=cuda_device, plant=("none",), seed=400 + len(case), **APPEND_CASES[case])
    _check(prob, seed=11)


def test_append_explicit_positions(cuda_device):
    prob = make_problem(name="pos", device=cuda_device, B=3, Hq=8, Hkv=2, d=128, r=32, M=64,
                        seq_lens=[700, 65, 1024], page_size=64, paged=True, kproj_fp8=True, plant=("none",), seed=431)
    _check(prob, seed=12, positions=torch.tensor([0, 63, 1023], dtype=torch.int32, device=cuda_device))


def test_append_then_decode_selects_the_new_token(cuda_device):
    # a new key aligned with the averaged query of its group is written by the append step and then
    # found by the index stage of the next decode
    prob = make_problem(name="loop", device=cuda_device, B=2, Hq=8, Hkv=2, d=128, r=32, M=64,
                        seq_lens=[3000, 900], page_size=64, paged=True, kproj_fp8=True, plant=("none",), seed=432)
    G = prob.G
    qbar = prob.q.float().view(prob.B, prob.Hkv, G, prob.d).mean(2)
    k_new = (qbar / qbar.norm(dim=-1, keepdim=True) * 40).to(torch.bfloat16)
    v_new = torch.zeros_like(k_new)
    _append(prob, k_new, v_new)
    ws = R.workspace(prob)
    idx, count = R.index_topm(prob, ws)
    for b in range(prob.B):
        n = int(prob.seq_lens[b])
        for h in range(prob.Hkv):
            assert n - 1 in idx[b, h, : int(count[b, h])].tolist()


def test_append_flags_bad_position_and_writes_nothing(cuda_device):
    prob = make_problem(name="bad", device=cuda_device, B=2, Hq=4, Hkv=1, d=64, r=16, M=16, seq_lens=[40, 20],
                        page_size=16, paged=True, kproj_fp8=True, plant=("none",), seed=433)
    k_new, v_new = _new_rows(prob, 13)
    before = _pools(prob)
    positions = torch.tensor([prob.max_seq_len, -1], dtype=torch.int32, device=cuda_device)
    ws = _append(prob, k_new, v_new, positions)
    assert L.lisa_check_device_error(ws) & L.DEVERR_INDEX
    after = _pools(prob)
    for name in ("k", "v", "kproj"):
        assert np.array_equal(after[name], before[name])


def test_append_full_size_128k(cuda_device):
    # the benchmark workload: 16 sequences x 8 KV heads at n = 131072; written rows checked against
    # the oracle for every (b, h), and a sample of other rows checked unchanged
    prob = config3(device=cuda_device, B=16)
    k_new, v_new = _new_rows(prob, 14)
    ps = prob.page_size
    lens = prob.seq_lens.cpu().numpy()
    table = prob.page_table.cpu().numpy()
    pages = [int(table[b][(lens[b] - 1) // ps]) for b in range(prob.B)]
    probe = [(pg, (int(lens[b]) - 1) % ps) for b, pg in enumerate(pages)]
    rng = np.random.default_rng(3)
    others = [(int(rng.integers(prob.num_pages)), int(rng.integers(ps))) for _ in range(64)]
    others = [o for o in others if o not in probe]
    def rows(sel):
        return {"k": [_bits16(prob.k_pool[pg, s]) for pg, s in sel], "v": [_bits16(prob.v_pool[pg, s]) for pg, s in sel],
                "kproj": [prob.kproj[pg, :, s].cpu().numpy() for pg, s in sel]}
    before_others = rows(others)
    ws = _append(prob, k_new, v_new)
    assert L.lisa_check_device_error(ws) == 0
    got = rows(probe)
    kb, vb = _bits16(k_new), _bits16(v_new)
    P = prob.P.cpu().numpy()
    scale = prob.kproj_scale.cpu().numpy()
    for b in range(prob.B):
        assert np.array_equal(got["k"][b], kb[b]) and np.array_equal(got["v"][b], vb[b])
        for h in range(prob.Hkv):
            c = O.project_key_fp32(P[h], O.bf16_to_f64(kb[b][h]))
            want = O.e4m3_encode((c / np.float32(scale[h])).astype(np.float32))
            assert np.array_equal(got["kproj"][b][h], want)
    after_others = rows(others)
    for name in ("k", "v", "kproj"):
        for x, y in zip(before_others[name], after_others[name]):
            assert np.array_equal(x, y)
