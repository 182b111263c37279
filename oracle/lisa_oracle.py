"""Plain fp64 CPU oracle for indexed sparse decode attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports, links or calls this
module; only the tests, the smoke check and the benchmark's CPU-baseline leg
do.  It shares no code with the CUDA path.  It is written for a reader who
checks it against the write-ups, not for speed.

Sources (cited by page and section; the pages carry no formulas, so each step
is the plain reading stated beside it):

* JSSA write-up, rit.work "jssa-sparse-attention-long-context" (article
  "Joint Subspace Sparse Attention for Efficient Long-Context Decoding"),
  section "Как JSSA сохраняет порядок токенов" (how JSSA keeps token order):
  per KV head a low-rank joint query/key subspace; at decode time the queries
  of one KV head are averaged, projected and every cached position is scored;
  after selection, attention is exact over the original full-size keys and
  values; the projected-key cache is FP8; each GQA group keeps its own index
  set; the kernel reads the selected positions straight from the cache.
* LISA write-ups (aikraft.ru "LISA: ускорение LLM на 50% без переобучения",
  section "Архитектура LISA"; opennieuws.be, section "Hybride architectuur
  voor efficiëntie"): a linear-attention branch runs beside the top-M sparse
  branch and the two are fused by a gate.
* IndexCache write-up (denisavetisyan.com, section "IndexCache: Совместное
  использование слоев для экстремального ускорения"): "Full" layers compute
  their top-k indices, "Shared" layers reuse those of the preceding Full layer.

Readings where the pages are silent (each is also listed with the design
notes): softmax scale 1/sqrt(d); "average" is the unweighted mean of the G
query heads; score = scale_h * <P_h qbar, c_t> with no extra nonlinearity;
FP8 is OCP E4M3 ("FN"); ties at the M-th score go to the lower position and
index sets are reported in ascending position order; n < M selects all n
positions; the linear branch uses phi = elu + 1, updates the state with the
current token before reading it, and the gate is
sigmoid(g) * sparse + (1 - sigmoid(g)) * linear per query head.

Every function here is pinned by tests/test_oracle_pins.py against something
other than itself (library decoders, dense attention, brute force, closed
forms, invariances).
"""

from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# Input decoding (bit-exact, to fp64)
# ---------------------------------------------------------------------------


def bf16_to_f64(bits) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> fp64.  bf16 is the top half of an IEEE fp32."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(bits) -> np.ndarray:
    """FP8 E4M3 codes (uint8) -> fp64, from the OCP 8-bit floating-point format.

    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.  Exponent field 0
    encodes subnormals m/8 * 2^-6.  There are no infinities; the codes with all
    exponent and mantissa bits set (0x7F, 0xFF) are NaN, so the largest finite
    magnitude is 1.75 * 2^8 = 448.
    """
    b = np.asarray(bits).astype(np.int64)
    sign = np.where((b & 0x80) != 0, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0**-6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 0xF) & (m == 7), np.nan, mag)
    return sign * mag


# ---------------------------------------------------------------------------
# The indexer (JSSA, "Как JSSA сохраняет порядок токенов", decoding paragraph)
# ---------------------------------------------------------------------------


def query_group_mean(q_rows: np.ndarray) -> np.ndarray:
    """Average of the G query vectors that share one KV head: [G][d] -> [d]."""
    return q_rows.sum(axis=0) / q_rows.shape[0]


def project_query(P: np.ndarray, qbar: np.ndarray) -> np.ndarray:
    """Project the averaged query into the head's r-dim subspace: u = P qbar, P is [r][d]."""
    return P @ qbar


def indexer_scores(u: np.ndarray, kproj_rows: np.ndarray, kproj_scale: float) -> np.ndarray:
    """Score of every cached position: s_t = scale_h * sum_i u_i * c_{t,i}.

    kproj_rows are the decoded projected keys [n][r]; kproj_scale is the
    per-head dequantisation factor of the FP8 cache (1 for an fp32 cache).
    """
    return kproj_scale * (kproj_rows @ u)


def select_top_m(scores: np.ndarray, M: int) -> np.ndarray:
    """The min(M, n) highest-scoring positions, in ascending position order.

    Order is by score descending, then by position ascending, so at a tie on
    the M-th score the lower position is kept.
    """
    n = scores.shape[0]
    m = min(M, n)
    pos = np.arange(n)
    order = np.lexsort((pos, -scores))  # primary: -score ascending; secondary: position
    return np.sort(order[:m])


# ---------------------------------------------------------------------------
# Exact attention over the selected set (JSSA: full-size keys and values)
# ---------------------------------------------------------------------------


def sparse_attention(q_rows: np.ndarray, k_rows: np.ndarray, v_rows: np.ndarray, softmax_scale: float):
    """Softmax attention of each query row over the given key/value rows.

    q_rows [G][d], k_rows/v_rows [m][d] -> (out [G][d], lse [G]) with
    lse = log sum_t exp(softmax_scale * q . k_t) (natural log).
    """
    logits = softmax_scale * (q_rows @ k_rows.T)  # [G][m]
    mx = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - mx)
    denom = w.sum(axis=1, keepdims=True)
    out = (w @ v_rows) / denom
    lse = (mx + np.log(denom))[:, 0]
    return out, lse


# ---------------------------------------------------------------------------
# LISA linear branch and gate ("Архитектура LISA" / "Hybride architectuur")
# ---------------------------------------------------------------------------


def phi(x: np.ndarray) -> np.ndarray:
    """Feature map elu(x) + 1: x + 1 for x > 0, exp(x) otherwise (always > 0)."""
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def linear_state_update(S: np.ndarray, z: np.ndarray, k_new: np.ndarray, v_new: np.ndarray):
    """Add the current token to the running state: S += phi(k) v^T, z += phi(k)."""
    fk = phi(k_new)
    return S + np.outer(fk, v_new), z + fk


def linear_read(S: np.ndarray, z: np.ndarray, q_rows: np.ndarray) -> np.ndarray:
    """Linear-attention output per query row: phi(q)^T S / (phi(q) . z)."""
    fq = phi(q_rows)
    return (fq @ S) / (fq @ z)[:, None]


def sigmoid(g: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-g))


def gate_combine(sparse_out: np.ndarray, lin_out: np.ndarray, gate_logits: np.ndarray) -> np.ndarray:
    """sigmoid(g) * sparse + (1 - sigmoid(g)) * linear, one logit per query row."""
    s = sigmoid(gate_logits)[:, None]
    return s * sparse_out + (1.0 - s) * lin_out


# ---------------------------------------------------------------------------
# One decode step over a paged batch
# ---------------------------------------------------------------------------


def _positions_to_rows(page_table_b: np.ndarray, page_size: int, pos: np.ndarray):
    return page_table_b[pos // page_size].astype(np.int64), (pos % page_size).astype(np.int64)


def head_scores(inp: dict, b: int, h: int) -> np.ndarray:
    """Indexer scores of every position of sequence b for KV head h (fp64)."""
    G = inp["Hq"] // inp["Hkv"]
    n = int(inp["seq_lens"][b])
    ps = inp["page_size"]
    q_rows = bf16_to_f64(inp["q"][b, h * G : (h + 1) * G])
    u = project_query(np.asarray(inp["P"][h], dtype=np.float64), query_group_mean(q_rows))
    pages, slots = _positions_to_rows(inp["page_table"][b], ps, np.arange(n))
    raw = inp["kproj"][pages, h, slots]  # [n][r]
    c = e4m3_to_f64(raw) if inp["kproj_fp8"] else np.asarray(raw, dtype=np.float64)
    return indexer_scores(u, c, float(inp["kproj_scale"][h]))


def head_attention(inp: dict, b: int, h: int, idx: np.ndarray):
    """Exact attention of KV head h's query group over positions idx of sequence b."""
    G = inp["Hq"] // inp["Hkv"]
    d = inp["d"]
    ps = inp["page_size"]
    scale = inp["softmax_scale"] if inp["softmax_scale"] > 0 else 1.0 / np.sqrt(d)
    q_rows = bf16_to_f64(inp["q"][b, h * G : (h + 1) * G])
    pages, slots = _positions_to_rows(inp["page_table"][b], ps, np.asarray(idx, dtype=np.int64))
    k_rows = bf16_to_f64(inp["k_pool"][pages, slots, h])
    v_rows = bf16_to_f64(inp["v_pool"][pages, slots, h])
    return sparse_attention(q_rows, k_rows, v_rows, scale)


def decode_step(inp: dict, reuse_idx=None, heads=None) -> dict:
    """Indexed sparse decode for every (b, KV head) pair (or the given subset).

    inp holds numpy arrays in the library's layouts (bf16 as uint16 bits, FP8
    as uint8 codes) plus the sizes; see workloads.synth for the layouts.
    reuse_idx[b][h], when given, is the index set of a Full layer that this
    (Shared) layer reuses instead of computing its own.  When inp has a "lin"
    entry the linear branch and the gate are applied.

    Returns idx[b][h] (ascending positions), scores[b][h] (fp64, only for
    computed sets), out [B][Hq][d] fp64, lse [B][Hq], and S/z after the update.
    """
    B, Hq, Hkv, d, M = inp["B"], inp["Hq"], inp["Hkv"], inp["d"], inp["M"]
    G = Hq // Hkv
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    idx = [[None] * Hkv for _ in range(B)]
    scores = [[None] * Hkv for _ in range(B)]
    out = np.full((B, Hq, d), np.nan)
    lse = np.full((B, Hq), np.nan)
    lin = inp.get("lin")
    S_new = None if lin is None else np.array(lin["S"], dtype=np.float64, copy=True)
    z_new = None if lin is None else np.array(lin["z"], dtype=np.float64, copy=True)
    for b, h in pairs:
        if reuse_idx is None:
            s = head_scores(inp, b, h)
            scores[b][h] = s
            sel = select_top_m(s, M)
        else:
            sel = np.asarray(reuse_idx[b][h], dtype=np.int64)
        idx[b][h] = sel
        o, l = head_attention(inp, b, h, sel)
        rows = slice(h * G, (h + 1) * G)
        if lin is not None:
            S2, z2 = linear_state_update(
                np.asarray(lin["S"][b, h], dtype=np.float64),
                np.asarray(lin["z"][b, h], dtype=np.float64),
                bf16_to_f64(lin["k_new"][b, h]),
                bf16_to_f64(lin["v_new"][b, h]),
            )
            S_new[b, h], z_new[b, h] = S2, z2
            lo = linear_read(S2, z2, bf16_to_f64(inp["q"][b, rows]))
            o = gate_combine(o, lo, np.asarray(lin["gate"][rows], dtype=np.float64))
        out[b, rows] = o
        lse[b, rows] = l
    return {"idx": idx, "scores": scores, "out": out, "lse": lse, "S": S_new, "z": z_new}


def layered_decode(layers: list, full_layers, heads=None) -> list:
    """IndexCache pattern: Full layers select, each Shared layer reuses the last Full layer's sets."""
    results = []
    last_full = None
    for layer, inp in enumerate(layers):
        if layer in full_layers:
            res = decode_step(inp, heads=heads)
            last_full = res["idx"]
        else:
            if last_full is None:
                raise ValueError("a Shared layer needs a preceding Full layer")
            res = decode_step(inp, reuse_idx=last_full, heads=heads)
        results.append(res)
    return results


# ---------------------------------------------------------------------------
# Append: the producer side of the caches (JSSA, "Как JSSA сохраняет порядок
# токенов": every cached position keeps a projected key in an FP8 cache beside
# the full-size keys and values)
# ---------------------------------------------------------------------------

# Non-negative finite E4M3 magnitudes in code order 0x00..0x7E (ascending).
_E4M3_MAGNITUDES = e4m3_to_f64(np.arange(0x7F))


def e4m3_encode(x) -> np.ndarray:
    """Values -> E4M3 codes (uint8): round to nearest, ties to the code with an even mantissa, and
    magnitudes of 448 and above saturate to 448 (the "satfinite" conversion of the OCP 8-bit format).

    The sign bit follows the sign of x, so -0.0 and small negatives that round to zero give 0x80.
    NaN gives 0xFF or 0x7F.  Candidates are the two representable neighbours of |x|.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    i = np.clip(np.searchsorted(_E4M3_MAGNITUDES, a, side="left"), 1, 0x7E)
    lo, hi = _E4M3_MAGNITUDES[i - 1], _E4M3_MAGNITUDES[i]
    take_hi = (a - lo > hi - a) | ((a - lo == hi - a) & ((i & 1) == 0))
    code = np.where(take_hi, i, i - 1)
    code = np.where(a >= 448.0, 0x7E, code)
    code = np.where(np.isnan(x), 0x7F, code)
    code = np.where(np.signbit(x), code | 0x80, code)
    return code.astype(np.uint8)


def project_key_fp32(P_h: np.ndarray, k: np.ndarray) -> np.ndarray:
    """c = P_h k in the fixed fp32 arithmetic of the append step: c_i starts at 0 and adds
    P_h[i][j] * k[j] for j = 0, 1, ..., d-1, with every product and every sum rounded to fp32
    (nearest even) separately.  P_h: [r][d], k: [d] (bf16 values, exact in fp32) -> [r] fp32.

    The pages fix no arithmetic for the projection; because the FP8 code is an integer decided by
    floating point, the oracle takes it in the same fp32 steps as the kernel.
    """
    P32 = np.asarray(P_h, dtype=np.float32)
    k32 = np.asarray(k, dtype=np.float32)
    c = np.zeros(P32.shape[0], dtype=np.float32)
    for j in range(P32.shape[1]):
        prod = (P32[:, j] * k32[j]).astype(np.float32)
        c = (c + prod).astype(np.float32)
    return c


def append_token(pools: dict, seq_lens, page_table, k_new_bits, v_new_bits, P, kproj_scale, kproj_fp8: bool,
                 positions=None) -> dict:
    """Write the current token of every (sequence b, KV head h) into copies of the caches.

    pools: "k", "v": uint16 bf16 bits [num_pages][ps][Hkv][d]; "kproj": uint8 codes or float32
    [num_pages][Hkv][ps][r].  k_new_bits/v_new_bits: uint16 [B][Hkv][d].  P: [Hkv][r][d] fp32.
    Position t_b = positions[b], else seq_lens[b] - 1; row = page_table[b][t // ps], slot t % ps.
    The K/V rows are copied bit for bit; the projected-key row is project_key_fp32(P_h, k), then
    for FP8 the code of (c / scale_h) rounded to fp32 and encoded by e4m3_encode.
    """
    out = {name: np.array(arr, copy=True) for name, arr in pools.items()}
    ps = out["k"].shape[1]
    B, Hkv = np.asarray(k_new_bits).shape[:2]
    for b in range(B):
        t = int(positions[b]) if positions is not None else int(seq_lens[b]) - 1
        page, slot = int(page_table[b][t // ps]), t % ps
        for h in range(Hkv):
            out["k"][page, slot, h] = k_new_bits[b][h]
            out["v"][page, slot, h] = v_new_bits[b][h]
            c = project_key_fp32(P[h], bf16_to_f64(k_new_bits[b][h]))
            if kproj_fp8:
                x = (c / np.float32(kproj_scale[h])).astype(np.float32)
                out["kproj"][page, h, slot] = e4m3_encode(x)
            else:
                out["kproj"][page, h, slot] = c
    return out


# ---------------------------------------------------------------------------
# Basis calibration (JSSA, "Как JSSA сохраняет порядок токенов": per head and
# layer, statistics of queries and keys are collected once and the basis is
# taken from eigenvectors of a matrix; the subspace is meant to preserve the
# query-key scores, not to reconstruct the vectors)
# ---------------------------------------------------------------------------


def calibration_matrix(q_samples: np.ndarray, k_samples: np.ndarray) -> np.ndarray:
    """C = (Q K + K Q) / 2 with Q = mean q q^T over the averaged group queries and K = mean k k^T.

    Reading (the pages name no matrix): for independent q and k, the expected product of the true
    score and the score through the projector Pi = P^T P is E[(q.k)(q.Pi k)] = tr(Pi K Q) =
    tr(Pi C); the rank-r projector maximising it spans the top-r eigenvectors of C.
    """
    q = np.asarray(q_samples, dtype=np.float64)
    k = np.asarray(k_samples, dtype=np.float64)
    Q = q.T @ q / q.shape[0]
    K = k.T @ k / k.shape[0]
    return 0.5 * (Q @ K + K @ Q)


def calibrate_basis(q_samples: np.ndarray, k_samples: np.ndarray, r: int):
    """P [r][d] (orthonormal rows, largest eigenvalue first) and its eigenvalues [r].

    Each row's sign is fixed so that its entry of largest magnitude is positive.
    """
    w, V = np.linalg.eigh(calibration_matrix(q_samples, k_samples))
    order = np.argsort(w)[::-1][:r]
    P = V[:, order].T.copy()
    for i in range(r):
        j = int(np.argmax(np.abs(P[i])))
        if P[i, j] < 0:
            P[i] = -P[i]
    return P, w[order]


# ---------------------------------------------------------------------------
# Multi-query indexer (several query tokens per sequence, e.g. speculative
# decoding): the same score per token, each token seeing the positions up to
# its own (causal)
# ---------------------------------------------------------------------------


def multi_query_scores(inp: dict, q_tokens, T: int, b: int, h: int) -> np.ndarray:
    """[T][n_b] fp64 indexer scores of the T query tokens q_tokens[b] ([T][Hq][d] bf16 bits) of
    sequence b for KV head h.  Token j sees positions t <= n_b - T + j; later entries are -inf."""
    n = int(inp["seq_lens"][b])
    out = np.full((T, n), -np.inf)
    for j in range(T):
        one = dict(inp)
        one["q"] = np.asarray(q_tokens)[:, j]  # [B][Hq][d]: token j of every sequence
        s = head_scores(one, b, h)
        lim = n - T + j
        if lim >= 0:  # a token of a sequence shorter than T may see no position at all
            out[j, : lim + 1] = s[: lim + 1]
    return out
