"""GPU parity of lisa_calibrate_basis (second moments + Jacobi eigen-decomposition) with the oracle.

Samples are drawn with a planted spectrum so that the top-r eigenvalues are well separated; then each
row of P must match the oracle's row (same sign convention) to fp32 accuracy, and the eigenvalues to
1e-4 relative.  The oracle computes in fp64 with a library eigensolver; the library in fp32 with its
own Jacobi solver."""

import numpy as np
import pytest
import torch

import indexed_top_sparse_b200 as L
from oracle import lisa_oracle as O

pytestmark = pytest.mark.gpu


def _samples(Hkv, n, d, seed, scale_fn):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(Hkv, n, d, generator=g)
    for h in range(Hkv):
        x[h] = x[h] * scale_fn(h, d)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("d,r", [(128, 32), (64, 16)])
def test_calibration_matches_oracle(cuda_device, d, r):
    Hkv, n = 4, 4096
    # well-separated leading spectrum: per-dimension scales decaying geometrically, rotated per head
    rot = [torch.linalg.qr(torch.randn(d, d, generator=torch.Generator().manual_seed(60 + h)))[0] for h in range(Hkv)]
    def qs(h, d):
        return torch.tensor(np.geomspace(3.0, 0.3, d), dtype=torch.float32)
    def ks(h, d):
        return torch.tensor(np.geomspace(2.5, 0.2, d), dtype=torch.float32)
    q = _samples(Hkv, n, d, 61, qs).float()
    k = _samples(Hkv, n, d, 62, ks).float()
    q = torch.stack([q[h] @ rot[h].T for h in range(Hkv)]).to(torch.bfloat16)
    k = torch.stack([k[h] @ rot[h].T for h in range(Hkv)]).to(torch.bfloat16)
    P = torch.full((Hkv, r, d), float("nan"), dtype=torch.float32, device=cuda_device)
    w = torch.full((Hkv, r), float("nan"), dtype=torch.float32, device=cuda_device)
    L.lisa_calibrate_basis(q.to(cuda_device).contiguous(), k.to(cuda_device).contiguous(), P, w)
    torch.cuda.synchronize()
    Pg, wg = P.cpu().double().numpy(), w.cpu().double().numpy()
    for h in range(Hkv):
        Po, wo = O.calibrate_basis(q[h].float().numpy(), k[h].float().numpy(), r)
        assert np.allclose(Pg[h] @ Pg[h].T, np.eye(r), atol=1e-5)
        assert np.allclose(wg[h], wo, rtol=1e-4)
        assert np.all(np.sum(Pg[h] * Po, axis=1) >= 1 - 1e-4)


def test_calibrated_basis_drives_the_decode_path(cuda_device):
    # P from lisa_calibrate_basis feeds the index stage; its selection matches the oracle's with
    # that P (the basis is an input of the decode step like any other)
    from tests.parity import check_index_sets
    from workloads import make_problem
    from workloads import run as R
    from workloads.host_view import host_inputs
    prob = make_problem(name="cal", device=cuda_device, B=2, Hq=8, Hkv=2, d=128, r=32, M=128,
                        seq_lens=[5000, 2000], page_size=64, paged=True, kproj_fp8=False, plant=("cosine", 0.01),
                        seed=540)
    G = prob.G
    qbar = prob.q.float().view(prob.B, prob.Hkv, G, prob.d).mean(2)  # [B][Hkv][d]
    qs = qbar.transpose(0, 1).contiguous().to(torch.bfloat16)  # [Hkv][B][d]
    n_k = 512
    ks = torch.stack([prob.k_pool[: n_k // prob.page_size, :, h].reshape(-1, prob.d) for h in range(prob.Hkv)])
    P = torch.empty(prob.Hkv, prob.r, prob.d, dtype=torch.float32, device=cuda_device)
    L.lisa_calibrate_basis(qs, ks.contiguous(), P)
    prob.P = P
    # projected keys of the cache under the new basis (fp32 cache, computed on the host in fp64)
    kp = torch.einsum("pshd,hrd->phsr", prob.k_pool.double(), P.double()).float()
    prob.kproj = kp.contiguous()
    ws = R.workspace(prob)
    idx, count = R.index_topm(prob, ws)
    inp = host_inputs(prob)
    ref = O.decode_step(inp)
    pairs = [(b, h) for b in range(prob.B) for h in range(prob.Hkv)]
    same = check_index_sets(idx.cpu().numpy(), count.cpu().numpy(), ref, inp["seq_lens"], prob.M, pairs)
    assert len(same) == len(pairs)
