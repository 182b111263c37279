"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against a library routine, a closed form, a
brute-force search, an invariance the method implies, or a hand-worked
example.  The mutation tests at the end plant plausible mistakes into a copy
of the oracle (on the CPU) and check that a pin catches each one.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lisa_oracle as O
from workloads import config1, make_problem
from workloads.host_view import host_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _expr(s):
    if isinstance(s, (int, float)):
        return float(s)
    return float(eval(s, {"__builtins__": {}}, {"e": math.e, "ln": math.log, "nan": math.nan}))


def _bf16_bits(x) -> np.ndarray:
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------
# Decoders
# ---------------------------------------------------------------------------


def test_e4m3_all_codes_match_library_decoder():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    # sign of zero
    assert math.copysign(1.0, ours[0x80]) == -1.0


def test_e4m3_golden_table():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "e4m3_codes.txt")) if ln.strip() and not ln.startswith("#")]
    assert len(rows) >= 15
    for code, val in rows:
        got = O.e4m3_to_f64(np.array([int(code, 16)], dtype=np.uint8))[0]
        want = _expr(val.replace("-0", "-0.0") if val == "-0" else val)
        if math.isnan(want):
            assert math.isnan(got), code
        else:
            assert got == want, (code, got, want)


def test_bf16_decode_matches_library():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2**16, size=50000, dtype=np.uint16)
    ours = O.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


# ---------------------------------------------------------------------------
# Indexer score
# ---------------------------------------------------------------------------


def _full_rank_problem(seed, fp8=False, Hkv=3, G=2, d=16, n=200, ps=16, paged=True):
    # r = d with an orthogonal (non-symmetric) basis: projected scores equal the
    # plain averaged-query logits  qbar . k_t  whatever the basis.
    return make_problem(
        name="pin", B=2, Hq=Hkv * G, Hkv=Hkv, d=d, r=d, M=8, seq_lens=[n, n - 37], page_size=ps,
        paged=paged, kproj_fp8=fp8, plant=("none",), seed=seed,
    )


def test_scores_full_rank_basis_equal_averaged_query_logits():
    prob = _full_rank_problem(7)
    inp = host_inputs(prob)
    G = prob.G
    for b in range(prob.B):
        n = int(prob.seq_lens[b])
        for h in range(prob.Hkv):
            s = O.head_scores(inp, b, h)
            # independent route: dense keys gathered by torch, mean query, torch matmul (fp64)
            t = torch.arange(n)
            pages = prob.page_table[b, t // prob.page_size].long()
            keys = prob.k_pool[pages, t % prob.page_size, h].to(torch.float64)
            qbar = prob.q[b, h * G : (h + 1) * G].to(torch.float64).mean(0)
            want = (keys @ qbar).numpy()
            # the projected-key cache was built in fp32, so agreement is to fp32 rounding
            assert np.allclose(s, want, rtol=1e-5, atol=1e-5 * np.abs(want).max())


def test_scores_fp8_path_reproduces_fp32_path_on_representable_keys():
    # Projected keys that lie exactly on the E4M3 grid (decoded by the library):
    # the FP8 path with a power-of-two scale must equal the fp32 path exactly.
    rng = np.random.default_rng(3)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    codes = rng.choice(finite, size=(50, 8)).astype(np.uint8)
    c_lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    u = rng.standard_normal(8)
    scale = 0.25
    s8 = O.indexer_scores(u, O.e4m3_to_f64(codes), scale)
    s32 = O.indexer_scores(u, c_lib * scale, 1.0)
    assert np.array_equal(s8, s32)
    # scores are linear in the per-head scale
    assert np.allclose(O.indexer_scores(u, O.e4m3_to_f64(codes), 2 * scale), 2 * s8)


# ---------------------------------------------------------------------------
# Top-M selection
# ---------------------------------------------------------------------------


def _brute_force_top_m(scores, M):
    """Best M-subset by exhaustive search: largest sum, then the lowest positions."""
    n = len(scores)
    best_sum, best = None, None
    for subset in itertools.combinations(range(n), min(M, n)):
        total = sum(scores[i] for i in subset)
        if best is None or total > best_sum or (total == best_sum and subset < best):
            best_sum, best = total, subset
    return list(best)


@pytest.mark.parametrize("seed", range(12))
def test_top_m_equals_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 11))
    scores = rng.integers(-3, 4, size=n).astype(np.float64)  # small integers: many exact ties
    for M in range(1, n + 2):
        got = O.select_top_m(scores, M).tolist()
        assert got == _brute_force_top_m(scores.tolist(), M), (scores, M)


def test_top_m_threshold_property_large():
    rng = np.random.default_rng(11)
    n, M = 20000, 700
    scores = np.round(rng.standard_normal(n), 2)  # coarse values: ties at the boundary
    sel = O.select_top_m(scores, M)
    assert len(sel) == M and np.all(np.diff(sel) > 0)
    chosen = np.zeros(n, bool)
    chosen[sel] = True
    thr = scores[sel].min()
    assert np.all(scores[~chosen] <= thr)
    # every tied position that was left out lies above every tied position kept
    tied_in = np.flatnonzero(chosen & (scores == thr))
    tied_out = np.flatnonzero(~chosen & (scores == thr))
    if len(tied_out):
        assert tied_in.max() < tied_out.min()


def test_top_m_when_context_shorter_than_budget():
    s = np.array([0.3, -1.0, 2.0])
    assert O.select_top_m(s, 5).tolist() == [0, 1, 2]


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------


def test_full_budget_equals_dense_attention():
    prob = make_problem(
        name="dense", B=2, Hq=8, Hkv=2, d=32, r=8, M=4096, seq_lens=[300, 129], page_size=16,
        paged=True, kproj_fp8=True, plant=("none",), seed=5,
    )
    inp = host_inputs(prob)
    res = O.decode_step(inp)
    G = prob.G
    for b in range(prob.B):
        n = int(prob.seq_lens[b])
        t = torch.arange(n)
        pages = prob.page_table[b, t // prob.page_size].long()
        for h in range(prob.Hkv):
            assert res["idx"][b][h].tolist() == list(range(n))
            k = prob.k_pool[pages, t % prob.page_size, h].to(torch.float64)
            v = prob.v_pool[pages, t % prob.page_size, h].to(torch.float64)
            q = prob.q[b, h * G : (h + 1) * G].to(torch.float64)
            want = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0]
            assert np.allclose(res["out"][b, h * G : (h + 1) * G], want.numpy(), rtol=1e-12, atol=1e-12)
            lse_want = torch.logsumexp((q @ k.T) / math.sqrt(prob.d), dim=1).numpy()
            assert np.allclose(res["lse"][b, h * G : (h + 1) * G], lse_want, rtol=1e-12, atol=1e-12)


def test_explicit_softmax_scale_is_used():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((3, 4))
    k = rng.standard_normal((5, 4))
    v = rng.standard_normal((5, 4))
    out, _ = O.sparse_attention(q, k, v, 0.37)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], scale=0.37
    )[0].numpy()
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12)


def _swap_positions(prob, b, t1, t2):
    """Swap two cached tokens of sequence b (keys, values and projected keys for every head)."""
    ps = prob.page_size
    p1, s1 = int(prob.page_table[b, t1 // ps]), t1 % ps
    p2, s2 = int(prob.page_table[b, t2 // ps]), t2 % ps
    for pool in (prob.k_pool, prob.v_pool):
        a, c = pool[p1, s1].clone(), pool[p2, s2].clone()
        pool[p1, s1], pool[p2, s2] = c, a
    a, c = prob.kproj[p1, :, s1].clone(), prob.kproj[p2, :, s2].clone()
    prob.kproj[p1, :, s1], prob.kproj[p2, :, s2] = c, a


def test_permuting_tokens_moves_only_positions():
    prob = make_problem(
        name="perm", B=1, Hq=4, Hkv=1, d=16, r=4, M=10, seq_lens=[120], page_size=8, paged=True,
        kproj_fp8=True, plant=("none",), seed=9,
    )
    base = O.decode_step(host_inputs(prob))
    sel = base["idx"][0][0].tolist()
    rest = [t for t in range(120) if t not in sel]
    # (1) swap two non-selected tokens: same set, same output
    _swap_positions(prob, 0, rest[3], rest[40])
    r1 = O.decode_step(host_inputs(prob))
    assert r1["idx"][0][0].tolist() == sel
    assert np.array_equal(r1["out"], base["out"])
    # (2) swap a selected token with a non-selected one: the set follows the token, output unchanged
    _swap_positions(prob, 0, sel[2], rest[7])
    r2 = O.decode_step(host_inputs(prob))
    want = sorted(set(sel) - {sel[2]} | {rest[7]})
    assert r2["idx"][0][0].tolist() == want
    assert np.allclose(r2["out"], base["out"], rtol=1e-12, atol=1e-13)


def test_selection_is_per_kv_head():
    prob = make_problem(
        name="heads", B=1, Hq=8, Hkv=4, d=16, r=4, M=12, seq_lens=[400], page_size=16, paged=False,
        kproj_fp8=True, plant=("none",), seed=13,
    )
    res = O.decode_step(host_inputs(prob))
    sets = [tuple(res["idx"][0][h]) for h in range(4)]
    assert len(set(sets)) == 4  # distinct groups choose their own tokens


def test_planted_keys_are_selected_on_config1():
    prob = config1()
    res = O.decode_step(host_inputs(prob))
    sel = set(res["idx"][0][0].tolist())
    planted = set(prob.planted[0][0].tolist())
    assert len(planted) == 8 and planted <= sel


# ---------------------------------------------------------------------------
# Linear branch and gate
# ---------------------------------------------------------------------------


def test_linear_recurrence_equals_parallel_form():
    rng = np.random.default_rng(21)
    n, d, G = 37, 8, 3
    k = rng.standard_normal((n, d))
    v = rng.standard_normal((n, d))
    q = rng.standard_normal((G, d))
    S, z = np.zeros((d, d)), np.zeros(d)
    for t in range(n):
        S, z = O.linear_state_update(S, z, k[t], v[t])
    got = O.linear_read(S, z, q)
    # parallel closed form with the library elu
    elu1 = lambda x: torch.nn.functional.elu(torch.tensor(x)) + 1.0
    a = elu1(q) @ elu1(k).T  # [G][n]
    want = (a @ torch.tensor(v)) / a.sum(1, keepdim=True)
    assert np.allclose(got, want.numpy(), rtol=1e-12, atol=1e-12)
    assert np.all(O.phi(rng.standard_normal(1000) * 30) > 0)


def test_gate_extremes():
    rng = np.random.default_rng(4)
    o, lin = rng.standard_normal((2, 5)), rng.standard_normal((2, 5))
    assert np.allclose(O.gate_combine(o, lin, np.array([60.0, 60.0])), o, atol=1e-20)
    assert np.allclose(O.gate_combine(o, lin, np.array([-60.0, -60.0])), lin, atol=1e-20)
    mid = O.gate_combine(o, lin, np.array([0.0, 0.0]))
    assert np.allclose(mid, 0.5 * (o + lin))


# ---------------------------------------------------------------------------
# Hand-worked example
# ---------------------------------------------------------------------------


def _golden_inputs(fx, with_lin):
    sz = fx["sizes"]
    ps, n = sz["page_size"], sz["n"]
    table = np.array([fx["page_table"]], dtype=np.int64)
    npages = table.max() + 1
    kproj = np.zeros((npages, 1, ps, sz["r"]))
    kpool = np.zeros((npages, ps, 1, sz["d"]), dtype=np.uint16)
    vpool = np.zeros((npages, ps, 1, sz["d"]), dtype=np.uint16)
    for t in range(n):
        p, s = table[0, t // ps], t % ps
        kproj[p, 0, s] = fx["kproj_by_position"][t]
        kpool[p, s, 0] = _bf16_bits(fx["k_by_position"][t])
        vpool[p, s, 0] = _bf16_bits(fx["v_by_position"][t])
    inp = {
        "B": 1, "Hq": sz["Hq"], "Hkv": 1, "d": sz["d"], "r": sz["r"], "M": sz["M"], "page_size": ps,
        "softmax_scale": fx["softmax_scale"], "seq_lens": np.array([n]), "page_table": table,
        "q": _bf16_bits(fx["q"])[None], "P": np.array([fx["P"]], dtype=np.float64), "kproj_fp8": False,
        "kproj": kproj, "kproj_scale": np.array([fx["kproj_scale"]]), "k_pool": kpool, "v_pool": vpool,
    }
    if with_lin:
        L = fx["linear"]
        inp["lin"] = {
            "S": np.array([[L["S"]]], dtype=np.float64), "z": np.array([[L["z"]]], dtype=np.float64),
            "k_new": _bf16_bits(L["k_new"])[None, None], "v_new": _bf16_bits(L["v_new"])[None, None],
            "gate": np.array([_expr(g) for g in L["gate"]]),
        }
    return inp


def test_hand_worked_decode_step():
    fx = json.load(open(os.path.join(GOLDEN, "tiny_decode.json")))
    res = O.decode_step(_golden_inputs(fx, with_lin=False))
    assert res["idx"][0][0].tolist() == fx["expected_idx"]
    assert np.allclose(res["scores"][0][0], [_expr(s) for s in fx["expected_scores"]], rtol=0, atol=1e-15)
    want = np.array([[_expr(x) for x in row] for row in fx["expected_out"]])
    assert np.allclose(res["out"][0], want, rtol=1e-14, atol=1e-14)
    assert np.allclose(res["lse"][0], [_expr(x) for x in fx["expected_lse"]], rtol=1e-14)


def test_hand_worked_decode_step_with_linear_branch():
    fx = json.load(open(os.path.join(GOLDEN, "tiny_decode.json")))
    res = O.decode_step(_golden_inputs(fx, with_lin=True))
    L = fx["linear"]
    assert np.allclose(res["S"][0, 0], [[_expr(x) for x in row] for row in L["expected_S"]])
    assert np.allclose(res["z"][0, 0], [_expr(x) for x in L["expected_z"]])
    want = np.array([[_expr(x) for x in row] for row in L["expected_out"]])
    assert np.allclose(res["out"][0], want, rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------------------
# Cross-layer reuse
# ---------------------------------------------------------------------------


def test_shared_layers_reuse_full_layer_sets():
    from workloads import config5

    lp = config5(layers=4, full_layers=(0, 2), B=1, Hq=4, Hkv=2, d=16, r=4, M=8, n=96)
    inps = [host_inputs(p) for p in lp.layers]
    res = O.layered_decode(inps, lp.full_layers)
    for layer in range(4):
        src = lp.source_layer(layer)
        for h in range(2):
            assert res[layer]["idx"][0][h].tolist() == res[src]["idx"][0][h].tolist()
    # a shared layer's output is its own attention over the reused set (not the source layer's output)
    o, _ = O.head_attention(inps[1], 0, 0, res[0]["idx"][0][0])
    lin = inps[1]["lin"]
    S2, z2 = O.linear_state_update(lin["S"][0, 0], lin["z"][0, 0], O.bf16_to_f64(lin["k_new"][0, 0]),
                                   O.bf16_to_f64(lin["v_new"][0, 0]))
    lo = O.linear_read(S2, z2, O.bf16_to_f64(inps[1]["q"][0, 0:2]))
    assert np.allclose(res[1]["out"][0, 0:2], O.gate_combine(o, lo, lin["gate"][0:2]))


# ---------------------------------------------------------------------------
# Mutation checks: a planted mistake in the oracle must trip a pin
# ---------------------------------------------------------------------------


def _expect_failure(monkeypatch, name, bad, test_fn, *args):
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        test_fn(*args)
    monkeypatch.undo()


# ---------------------------------------------------------------------------
# Append step: E4M3 encoder, fixed fp32 projection, cache writes
# ---------------------------------------------------------------------------


def test_e4m3_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(O.e4m3_encode(O.e4m3_to_f64(codes)), codes)


def test_e4m3_encode_matches_library_conversion():
    # torch's float8_e4m3fn conversion: round to nearest even within the finite range
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(0, 40, 50000), rng.normal(0, 0.01, 20000), rng.uniform(-448, 448, 20000)])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x.astype(np.float64)), ref)


def test_e4m3_encode_ties_and_saturation():
    mags = O.e4m3_to_f64(np.arange(0x7F))
    for c in range(0x7E):  # midpoint between codes c and c + 1 goes to the even one
        mid = (mags[c] + mags[c + 1]) / 2
        want = c if c % 2 == 0 else c + 1
        assert int(O.e4m3_encode(mid)) == want and int(O.e4m3_encode(-mid)) == want | 0x80
    assert int(O.e4m3_encode(448.0)) == 0x7E and int(O.e4m3_encode(449.0)) == 0x7E
    assert int(O.e4m3_encode(1e30)) == 0x7E and int(O.e4m3_encode(-1e30)) == 0xFE
    assert int(O.e4m3_encode(-0.0)) == 0x80 and int(O.e4m3_encode(0.0)) == 0x00


def test_fp32_projection_is_sequential_and_within_rounding_of_exact():
    rng = np.random.default_rng(6)
    P = rng.normal(0, 1, (32, 128)).astype(np.float32)
    k = O.bf16_to_f64(_bf16_bits(rng.normal(0, 1, 128)))
    c = O.project_key_fp32(P, k)
    exact = P.astype(np.float64) @ k
    bound = 128 * 2.0**-23 * (np.abs(P.astype(np.float64)) @ np.abs(k))
    assert np.all(np.abs(c.astype(np.float64) - exact) <= bound)
    # the fixed order: sequential left-to-right fp32 sums, checked on a case where order matters
    P2 = np.array([[1.0, 2.0**-24, 2.0**-24, -1.0]], dtype=np.float32)
    k2 = np.ones(4)
    assert O.project_key_fp32(P2, k2)[0] == np.float32(0.0)  # (1 + 2^-24) rounds to 1 twice, then - 1
    # integers are exact in any order
    P3 = rng.integers(-8, 8, (16, 64)).astype(np.float32)
    k3 = rng.integers(-8, 8, 64).astype(np.float64)
    assert np.array_equal(O.project_key_fp32(P3, k3), (P3.astype(np.float64) @ k3).astype(np.float32))


def test_append_writes_exactly_the_current_rows():
    rng = np.random.default_rng(7)
    pages, ps, Hkv, d, r, B = 6, 16, 2, 64, 16, 3
    pools = {"k": rng.integers(0, 65535, (pages, ps, Hkv, d)).astype(np.uint16),
             "v": rng.integers(0, 65535, (pages, ps, Hkv, d)).astype(np.uint16),
             "kproj": rng.integers(0, 255, (pages, Hkv, ps, r)).astype(np.uint8)}
    seq_lens = [20, 1, 33]
    page_table = [[4, 1, 0], [5, 2, 3], [2, 0, 3]]
    kb = _bf16_bits(rng.normal(0, 1, (B, Hkv, d)))
    vb = _bf16_bits(rng.normal(0, 1, (B, Hkv, d)))
    P = rng.normal(0, 1, (Hkv, r, d)).astype(np.float32)
    scale = np.array([0.05, 0.02], dtype=np.float32)
    out = O.append_token(pools, seq_lens, page_table, kb, vb, P, scale, True)
    touched = {(page_table[b][(seq_lens[b] - 1) // ps], (seq_lens[b] - 1) % ps) for b in range(B)}
    for page in range(pages):
        for slot in range(ps):
            same = (page, slot) not in touched
            assert np.array_equal(out["k"][page, slot], pools["k"][page, slot]) == same
            assert np.array_equal(out["kproj"][page, :, slot], pools["kproj"][page, :, slot]) == same
    b = 2  # position 32 -> page_table[2][2] = 3, slot 0
    assert np.array_equal(out["k"][3, 0], kb[b]) and np.array_equal(out["v"][3, 0], vb[b])
    for h in range(Hkv):
        x = (P[h].astype(np.float64) @ O.bf16_to_f64(kb[b][h])) / scale[h]
        dec = O.e4m3_to_f64(out["kproj"][3, h, 0])
        sat = np.abs(x) >= 448
        assert np.all(dec[sat] == np.sign(x[sat]) * 448)  # saturated to the largest finite magnitude
        # otherwise within half an E4M3 step (2^-4 relative, 2^-10 absolute among subnormals)
        assert np.all(np.abs(dec - x)[~sat] <= np.maximum(np.abs(x) * 2.0**-4, 2.0**-10)[~sat] * 1.001)
        assert sat.any() or h == 0
    out2 = O.append_token(pools, seq_lens, page_table, kb, vb, P, scale, True, positions=[0, 0, 0])
    assert np.array_equal(out2["k"][4, 0], kb[0]) and np.array_equal(out2["k"][2, 0], kb[2])


# ---------------------------------------------------------------------------
# Basis calibration
# ---------------------------------------------------------------------------


def _orthonormal(rng, r, d):
    return np.linalg.qr(rng.normal(size=(d, r)))[0].T


def test_calibration_with_isotropic_queries_is_key_pca():
    # Q = I (queries = sqrt(d) times an orthogonal matrix): the basis is the keys' principal subspace,
    # taken here from the SVD of the key samples
    rng = np.random.default_rng(8)
    d, r = 64, 16
    q = np.sqrt(d) * np.linalg.qr(rng.normal(size=(d, d)))[0]
    k = rng.normal(size=(3000, d)) * np.linspace(4, 0.2, d)
    P, _ = O.calibrate_basis(q, k, r)
    Vt = np.linalg.svd(k, full_matrices=False)[2][:r]
    assert np.allclose(P.T @ P, Vt.T @ Vt, atol=1e-8)


def test_calibration_diagonal_moments_pick_largest_products():
    d, r = 32, 8
    a = np.linspace(1, 2, d)[::-1] ** 2
    b = np.roll(np.linspace(0.5, 3, d), 11) ** 2
    q = np.diag(np.sqrt(a * d))  # Q = diag(a)
    k = np.diag(np.sqrt(b * d))  # K = diag(b)
    P, w = O.calibrate_basis(q, k, r)
    top = np.argsort(a * b)[::-1][:r]
    assert np.allclose(np.abs(P), np.eye(d)[top], atol=1e-12) and np.all(P[np.arange(r), top] > 0)
    assert np.allclose(w, (a * b)[top])


def test_calibration_maximises_the_score_agreement():
    # brute force over all sample pairs: mean of (q.k)(q.P^T P k) equals tr(P C P^T), and the
    # calibrated basis beats random orthonormal bases on it
    rng = np.random.default_rng(9)
    d, r = 32, 6
    q = rng.normal(size=(300, d)) @ np.diag(np.linspace(2, 0.5, d))
    k = rng.normal(size=(400, d)) @ np.diag(np.linspace(0.3, 2.5, d))
    P, w = O.calibrate_basis(q, k, r)
    def agreement(B):
        S = q @ k.T
        Sp = (q @ B.T) @ (B @ k.T)
        return float(np.mean(S * Sp))
    C = O.calibration_matrix(q, k)
    assert np.isclose(agreement(P), np.trace(P @ C @ P.T), rtol=1e-10)
    assert np.isclose(agreement(P), float(np.sort(np.linalg.eigvalsh(C))[::-1][:r].sum()), rtol=1e-10)
    best_random = max(agreement(_orthonormal(rng, r, d)) for _ in range(200))
    assert agreement(P) > best_random
    assert np.allclose(P @ P.T, np.eye(r), atol=1e-12)


# ---------------------------------------------------------------------------
# Multi-query indexer
# ---------------------------------------------------------------------------


def test_multi_query_scores_are_single_queries_over_causal_prefixes():
    # token j of T equals a one-token decode of the same sequence cut to n - T + j + 1 positions
    prob = make_problem(name="mq", B=2, Hq=8, Hkv=2, d=64, r=16, M=16, seq_lens=[300, 40], page_size=16, paged=True,
                        kproj_fp8=True, plant=("none",), seed=30, device=torch.device("cpu"))
    inp = host_inputs(prob)
    T = 3
    rng = np.random.default_rng(31)
    qt = _bf16_bits(rng.normal(size=(prob.B, T, prob.Hq, prob.d)))
    for b in range(prob.B):
        n = int(inp["seq_lens"][b])
        for h in range(prob.Hkv):
            s = O.multi_query_scores(inp, qt, T, b, h)
            for j in range(T):
                one = dict(inp)
                one["q"] = qt[:, j]
                one["seq_lens"] = np.array(inp["seq_lens"]).copy()
                one["seq_lens"][b] = n - T + j + 1
                ref = O.head_scores(one, b, h)
                assert np.allclose(s[j, : n - T + j + 1], ref, rtol=1e-12, atol=1e-12)
                assert np.all(np.isneginf(s[j, n - T + j + 1 :]))


def test_multi_query_tokens_of_a_short_sequence_see_only_their_prefix():
    # n = 2 positions, T = 4 tokens: tokens 0 and 1 see nothing, token 2 sees position 0, token 3 both
    prob = make_problem(name="mq", B=1, Hq=4, Hkv=1, d=64, r=16, M=4, seq_lens=[2], page_size=16, paged=False,
                        kproj_fp8=True, plant=("none",), seed=32, device=torch.device("cpu"))
    inp = host_inputs(prob)
    rng = np.random.default_rng(33)
    qt = _bf16_bits(rng.normal(size=(1, 4, prob.Hq, prob.d)))
    s = O.multi_query_scores(inp, qt, 4, 0, 0)
    assert s.shape == (4, 2)
    assert np.all(np.isneginf(s[0])) and np.all(np.isneginf(s[1]))
    assert np.isfinite(s[2, 0]) and np.isneginf(s[2, 1])
    assert np.all(np.isfinite(s[3]))


def test_mutations_are_caught(monkeypatch):
    good_project, good_select, good_attn = O.project_query, O.select_top_m, O.sparse_attention
    good_gate, good_upd = O.gate_combine, O.linear_state_update
    # transposed basis
    _expect_failure(monkeypatch, "project_query", lambda P, q: P.T @ q,
                    test_scores_full_rank_basis_equal_averaged_query_logits)
    # summed instead of averaged query group
    _expect_failure(monkeypatch, "query_group_mean", lambda q: q.sum(0),
                    test_scores_full_rank_basis_equal_averaged_query_logits)
    # tie broken towards the higher position
    def bad_select(s, M):
        n = len(s)
        order = np.lexsort((-np.arange(n), -s))
        return np.sort(order[: min(M, n)])
    monkeypatch.setattr(O, "select_top_m", bad_select)
    caught = 0
    for seed in range(12):
        try:
            test_top_m_equals_brute_force_with_ties(seed)
        except AssertionError:
            caught += 1
    monkeypatch.undo()
    assert caught > 0
    # softmax scale dropped
    _expect_failure(monkeypatch, "sparse_attention", lambda q, k, v, s: good_attn(q, k, v, 1.0),
                    test_full_budget_equals_dense_attention)
    # gate weights swapped
    _expect_failure(monkeypatch, "gate_combine", lambda o, l, g: good_gate(l, o, g), test_gate_extremes)
    # linear read before the update (current token missing)
    _expect_failure(monkeypatch, "linear_state_update", lambda S, z, k, v: (S, z),
                    test_hand_worked_decode_step_with_linear_branch)
    # encoder: ties away from zero instead of to even
    good_enc = O.e4m3_encode
    def enc_ties_up(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.abs(x)
        i = np.clip(np.searchsorted(O._E4M3_MAGNITUDES, a, side="left"), 1, 0x7E)
        lo, hi = O._E4M3_MAGNITUDES[i - 1], O._E4M3_MAGNITUDES[i]
        code = np.where(a - lo >= hi - a, i, i - 1)
        code = np.where(a >= 448.0, 0x7E, code)
        return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)
    _expect_failure(monkeypatch, "e4m3_encode", enc_ties_up, test_e4m3_encode_ties_and_saturation)
    # projection summed in fp64 (order and rounding not the fixed ones)
    _expect_failure(monkeypatch, "project_key_fp32",
                    lambda P, k: (np.asarray(P, np.float64) @ np.asarray(k, np.float64)).astype(np.float32),
                    test_fp32_projection_is_sequential_and_within_rounding_of_exact)
    assert O.e4m3_encode is good_enc
    # calibration matrix taken from the keys alone (plain key PCA)
    good_cal = O.calibration_matrix
    _expect_failure(monkeypatch, "calibration_matrix",
                    lambda q, k: np.asarray(k, np.float64).T @ np.asarray(k, np.float64) / len(k),
                    test_calibration_diagonal_moments_pick_largest_products)
    assert O.calibration_matrix is good_cal
    # multi-query causal limit off by one (token j seeing one position too few)
    good_mq = O.multi_query_scores
    def mq_short(inp, q_tokens, T, b, h):
        out = good_mq(inp, q_tokens, T, b, h)
        n = int(inp["seq_lens"][b])
        for j in range(T):
            out[j, n - T + j] = -np.inf
        return out
    _expect_failure(monkeypatch, "multi_query_scores", mq_short,
                    test_multi_query_scores_are_single_queries_over_causal_prefixes)
    assert O.multi_query_scores is good_mq
    assert O.project_query is good_project and O.select_top_m is good_select and O.linear_state_update is good_upd
