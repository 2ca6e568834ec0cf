"""CPU oracle for AQUA's online attention step.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this module.  The product (the CUDA library and its Python
binding) never imports, links or executes anything here, and this module
imports nothing from the product.

What it follows.  AQUA (Attention via QUery mAgnitudes, arXiv 2509.11155):
  * page "AQUA: Attention via QUery mAgnitudes for Memory and Compute Efficient
    Inference in LLMs" (shd-paper digest), sections "技术框架" (technical
    framework) and "关键设计" (key design), and its original-language abstract;
  * blog "AQUA (Attention via QUery mAgnitudes)" (edgentiq), sections
    "How AQUA Works: A Two-Phase Approach" and "AQUA-Memory: Dual Savings".
The pages print no formula, listing or worked example.  Each function states
the reading it takes where the pages are silent; the workload statement that
accompanies the pages fixes the 1/sqrt(d) scale, ties to the lower index and
the unprojected V.

Precision.  Everything is float64.  Two roundings are part of the defined
result because they are storage formats, not arithmetic choices: projected
keys are stored in the cache's element type (bf16 round-to-nearest-even, or
fp32), and a bf16 output tensor holds the RNE rounding of the exact output.
The oracle implements both roundings itself (``round_bf16``).

Pins (what fixes each function other than itself) live in
tests/test_oracle_pins.py.  Every function here is pinned.  The pages print
no formula for ``breakeven_length``; it is pinned against a multiply-add
count of this module's own ``project`` and ``sparse_scores``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


# ----------------------------------------------------------------------------
# storage roundings
# ----------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), as float64.

    bf16 keeps 8 significant bits and float32's exponent range: a value in
    [2^e, 2^(e+1)) is rounded to a multiple of 2^(e-7); below the smallest
    normal exponent (-126) the spacing stays 2^-133.  Values beyond the largest
    finite bf16 become +-inf.  Rounding is done directly from float64, never
    through float32, so no double rounding occurs.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    fin = np.isfinite(x) & (x != 0)
    xv = x[fin]
    _, ex = np.frexp(np.abs(xv))          # |x| = m * 2^ex, m in [0.5, 1)
    e = ex - 1                            # |x| in [2^e, 2^(e+1))
    q = np.maximum(e, -126) - 7           # exponent of the bf16 spacing
    r = np.ldexp(np.round(np.ldexp(xv, -q)), q)   # np.round: half to even
    max_bf16 = np.ldexp(np.float64(0xFF), 120)    # (2 - 2^-7) * 2^127
    r = np.where(np.abs(r) > max_bf16, np.copysign(np.inf, r), r)
    out[fin] = r
    return out


def store(x, dtype: str) -> np.ndarray:
    """Value of x once stored in a cache/output of element type dtype ('bf16'|'f32'|'f64')."""
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------
# offline step: calibration
# ----------------------------------------------------------------------------

def calibrate(X) -> tuple[np.ndarray, np.ndarray]:
    """Offline projection P from a calibration matrix X [n, d].

    "Offline Projection Computation" (edgentiq, How AQUA Works) / abstract:
    SVD of the calibration data; P holds the right singular vectors as
    columns, ordered by descending singular value.  X stacks calibration
    queries and keys and is not centred (SVD, not PCA).  Column signs are
    arbitrary; neither selection (by |.|) nor q~.k~ depends on them.
    Returns (P [d, d], sigma [d]).
    """
    X = np.asarray(X, dtype=np.float64)
    _, sigma, vt = np.linalg.svd(X, full_matrices=False)
    return vt.T.copy(), sigma


# ----------------------------------------------------------------------------
# online step
# ----------------------------------------------------------------------------

def project(x, P) -> np.ndarray:
    """x~ = x P for row vectors x [..., d] (abstract: queries and keys are projected by P)."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(P, dtype=np.float64)


def select_dims(qt, k: int, m: int | None = None) -> np.ndarray:
    """Indices S of the k largest |q~_j| among j < m, ascending.

    The abstract has each query keep a sparse, query-dependent subset of
    dimensions chosen by magnitude; the blog (edgentiq, Online Inference)
    takes the dimensions where the projected query is largest.  Magnitude reading:
    |q~_j|.  Equal magnitudes go to the lower index.  With a truncated cache
    (AQUA-Memory) only the m stored dimensions are candidates.
    """
    qt = np.asarray(qt, dtype=np.float64)
    d = qt.shape[-1]
    m = d if m is None else m
    if not (1 <= k <= m <= d):
        raise ValueError(f"need 1 <= k <= m <= d, got k={k} m={m} d={d}")
    mag = np.abs(qt[:m])
    order = np.lexsort((np.arange(m), -mag))   # by -|q~| then by index
    return np.sort(order[:k])


def sparse_scores(qt, S, Kt, scale: float) -> np.ndarray:
    """s_t = scale * sum_{j in S} q~_j K~[t, j]  (scores on the selected dimensions only)."""
    S = np.asarray(S)
    return (np.asarray(Kt, dtype=np.float64)[:, S] @ np.asarray(qt, dtype=np.float64)[S]) * scale


def softmax(s) -> tuple[np.ndarray, float]:
    """Softmax over the visible tokens; also returns lse = log(sum(exp(s)))."""
    s = np.asarray(s, dtype=np.float64)
    mx = np.max(s)
    e = np.exp(s - mx)
    z = e.sum()
    return e / z, float(mx + np.log(z))


def attend_one(qt, k: int, Kt, V, scale: float, m: int | None = None):
    """One query head over T visible tokens: (o [d], probs [T], lse, S).

    Scores on the selected dimensions, softmax, weighted sum of the
    unprojected values V [T, d].
    """
    S = select_dims(qt, k, m)
    if len(Kt) == 0:
        # no visible token: the weighted sum is empty (zero) and log(sum exp) = -inf
        return np.zeros(np.shape(V)[-1]), np.zeros(0), -np.inf, S
    s = sparse_scores(qt, S, Kt, scale)
    p, lse = softmax(s)
    return p @ np.asarray(V, dtype=np.float64), p, lse, S


def default_scale(d: int) -> float:
    """1/sqrt(d) with d the full head dimension (reduces to standard attention at k = d)."""
    return 1.0 / np.sqrt(d)


# ----------------------------------------------------------------------------
# cache building and the decode / prefill steps
# ----------------------------------------------------------------------------
#
# AQUA-Memory on the values.  The edgentiq blog ("AQUA-Memory: Dual Savings")
# says the lowest-importance dimensions are dropped before the key AND value
# vectors are stored.  The pages give no formula; the plainest reading, taken
# here: values are projected by the same orthogonal P as the keys of their KV
# head, the first m_v projected dimensions are stored, V^ = store((v P)[:m_v]),
# and the attention output is brought back to the value space by the
# transpose of those columns, o = (sum_t p_t V^_t) P[:, :m_v]^T.  With m_v = d
# this is exactly the unpruned output (P P^T = I); for m_v < d it is the
# unpruned output projected onto the span of P's first m_v columns (up to the
# storage rounding of V^).  Without v_projected the values are unprojected,
# as the workload statement asks for the main path.

def build_key_cache(k, P, kv_dtype: str, m: int | None = None) -> np.ndarray:
    """Projected-key cache K~ = store(k P)[..., :m] for keys k [..., Hkv, d] and P [Hkv, d, d].

    AQUA-Memory (edgentiq, "AQUA-Memory: Dual Savings"): the static pruning
    drops the lowest-importance projected dimensions before caching; reading:
    those are the trailing ones (smallest singular values), so the first m are
    kept.  The cache is token-major here for readability.
    """
    k = np.asarray(k, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    Hkv, d = k.shape[-2], k.shape[-1]
    m = d if m is None else m
    kt = np.einsum("...gi,gij->...gj", k, P)
    return store(kt[..., :m], kv_dtype)


def build_value_cache(v, P, kv_dtype: str, m_v: int | None = None) -> np.ndarray:
    """Pruned projected-value cache V^ = store((v P)[..., :m_v]) for values v [..., Hkv, d].

    AQUA-Memory on the values (see the reading above): same P as the keys of
    the KV head, the first m_v projected dimensions kept.
    """
    v = np.asarray(v, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    m_v = v.shape[-1] if m_v is None else m_v
    vt = np.einsum("...gi,gij->...gj", v, P)
    return store(vt[..., :m_v], kv_dtype)


def unproject_values(o_hat, P_g) -> np.ndarray:
    """o = o^ P[:, :m_v]^T: an output over the m_v stored projected value
    dimensions, brought back to the d value dimensions."""
    o_hat = np.asarray(o_hat, dtype=np.float64)
    m_v = o_hat.shape[-1]
    return o_hat @ np.asarray(P_g, dtype=np.float64)[:, :m_v].T


def decode(q, P, Kt, V, lens, k: int, scale: float | None = None, m: int | None = None,
           out_dtype: str = "f64", v_projected: bool = False):
    """One AQUA decode step for every (sequence, query head).

    q   [B, Hq, d]          queries (their new keys are already in the cache);
    P   [Hkv, d, d]         projection per KV head (query head h uses P[h // G]);
    Kt  [B, Hkv, T, m]      projected-key cache (token-major), T >= lens[b];
    V   [B, Hkv, T, d]      unprojected values, or with v_projected the pruned
                            projected values V^ [B, Hkv, T, m_v] (build_value_cache);
    lens[B]                 visible tokens per sequence.
    Returns dict: out [B, Hq, d], sel [B, Hq, k], qt [B, Hq, d], lse [B, Hq],
    probs list-of-lists [b][h] -> [lens[b]].
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = Kt.shape[1]
    G = Hq // Hkv
    m = Kt.shape[-1] if m is None else m
    scale = default_scale(d) if scale is None else scale
    out = np.zeros((B, Hq, d))
    sel = np.zeros((B, Hq, k), dtype=np.int64)
    qts = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    probs = [[None] * Hq for _ in range(B)]
    for b in range(B):
        T = int(lens[b])
        for h in range(Hq):
            g = h // G
            qt = project(q[b, h], P[g])
            o, p, l, S = attend_one(qt, k, Kt[b, g, :T], V[b, g, :T], scale, m)
            if v_projected:
                o = unproject_values(o, P[g])
            out[b, h], sel[b, h], qts[b, h], lse[b, h], probs[b][h] = o, S, qt, l, p
    if out_dtype == "bf16":
        out = round_bf16(out)
    elif out_dtype == "f32":
        out = store(out, "f32")
    return {"out": out, "sel": sel, "qt": qts, "lse": lse, "probs": probs}


def prefill(q, pos0: int, P, Kt, V, k: int, scale: float | None = None, m: int | None = None,
            out_dtype: str = "f64", v_projected: bool = False):
    """Causal AQUA attention for a chunk of queries at absolute positions pos0 .. pos0+L-1.

    q [L, Hq, d]; Kt [Hkv, >= pos0+L, m]; V [Hkv, >= pos0+L, d] (one sequence),
    or with v_projected the pruned projected values [Hkv, >= pos0+L, m_v].
    Row i sees tokens 0 .. pos0+i.  Each (row, head) selects its own k
    dimensions, exactly as a decode step at that position would.
    Returns (out [L, Hq, d], sel [L, Hq, k]).
    """
    q = np.asarray(q, dtype=np.float64)
    L, Hq, d = q.shape
    Hkv = Kt.shape[0]
    G = Hq // Hkv
    m = Kt.shape[-1] if m is None else m
    scale = default_scale(d) if scale is None else scale
    out = np.zeros((L, Hq, d))
    sel = np.zeros((L, Hq, k), dtype=np.int64)
    for i in range(L):
        T = pos0 + i + 1
        for h in range(Hq):
            g = h // G
            qt = project(q[i, h], P[g])
            o, _, _, S = attend_one(qt, k, Kt[g, :T], V[g, :T], scale, m)
            if v_projected:
                o = unproject_values(o, P[g])
            out[i, h], sel[i, h] = o, S
    if out_dtype == "bf16":
        out = round_bf16(out)
    elif out_dtype == "f32":
        out = store(out, "f32")
    return out, sel


# ----------------------------------------------------------------------------
# H2O heavy-hitter eviction on top of AQUA
# ----------------------------------------------------------------------------
#
# The pages only name H2O (the abstract says AQUA combines with token eviction
# methods such as H2O and speeds them up).  Reading taken (the plainest H2O rule):
#   * per (sequence, KV head) a set of at most `budget` cached tokens;
#   * each token carries a cumulative score: the sum, over the G query heads
#     of its group and over every decode step since it entered, of its AQUA
#     softmax probability; a new token starts with its own current-step value;
#   * after each append, if the set holds more than `budget` tokens, exactly one
#     is evicted: the lowest score among tokens outside the `recent` most
#     recent positions, ties to the oldest position.

def h2o_choose_victim(score, pos, t_newest: int, recent: int) -> int:
    """Index of the token to evict: min score among pos <= t_newest - recent, ties -> oldest.

    Returns -1 when no token is outside the recent window.
    """
    score = np.asarray(score)
    pos = np.asarray(pos)
    best = -1
    for i in range(len(pos)):
        if pos[i] > t_newest - recent:
            continue
        if best < 0 or score[i] < score[best] or (score[i] == score[best] and pos[i] < pos[best]):
            best = i
    return best


@dataclass
class H2OSeq:
    """Retained tokens of one (sequence, KV head): positions, scores, K~ rows, V rows."""
    pos: list = field(default_factory=list)
    score: list = field(default_factory=list)
    kt: list = field(default_factory=list)
    v: list = field(default_factory=list)


def h2o_decode_step(seqs, q_b, k_new_b, v_new_b, t_abs: int, P, k: int, budget: int, recent: int,
                    kv_dtype: str, m: int | None = None, scale: float | None = None, m_v: int | None = None):
    """One decode step of one sequence with H2O eviction.

    seqs: list over KV heads of H2OSeq (modified in place); q_b [Hq, d];
    k_new_b, v_new_b [Hkv, d]; the new token has absolute position t_abs.
    With m_v the values are kept as pruned projected values (AQUA-Memory on
    the values; the retained rows in seqs are then V^ rows).
    Returns out [Hq, d] (float64) and the evicted positions per KV head.
    """
    q_b = np.asarray(q_b, dtype=np.float64)
    Hq, d = q_b.shape
    Hkv = len(seqs)
    G = Hq // Hkv
    m = d if m is None else m
    scale = default_scale(d) if scale is None else scale
    out = np.zeros((Hq, d))
    evicted = []
    for g in range(Hkv):
        s = seqs[g]
        kt_new = store(project(k_new_b[g], P[g])[:m], kv_dtype)
        s.pos.append(t_abs)
        s.score.append(0.0)
        s.kt.append(kt_new)
        if m_v is None:
            s.v.append(np.asarray(v_new_b[g], dtype=np.float64))
        else:
            s.v.append(store(project(v_new_b[g], P[g])[:m_v], kv_dtype))
        Kt = np.array(s.kt)
        Vv = np.array(s.v)
        acc = np.zeros(len(s.pos))
        for h in range(g * G, (g + 1) * G):
            qt = project(q_b[h], P[g])
            o, p, _, _ = attend_one(qt, k, Kt, Vv, scale, m)
            out[h] = o if m_v is None else unproject_values(o, P[g])
            acc += p
        for i in range(len(s.pos)):
            s.score[i] += acc[i]
        ev = -1
        if len(s.pos) > budget:
            ev = h2o_choose_victim(s.score, s.pos, t_abs, recent)
            if ev >= 0:
                evicted.append(s.pos[ev])
                for lst in (s.pos, s.score, s.kt, s.v):
                    del lst[ev]
        if ev < 0:
            evicted.append(-1)
    return out, evicted


# ----------------------------------------------------------------------------
# magnitude selection versus slicing off the first dimensions
# ----------------------------------------------------------------------------
#
# The edgentiq blog ("Validation and Generalizability") reports that choosing
# the dimensions by the query's magnitude loses about half the information that
# keeping a fixed leading block of dimensions loses.  It gives no formula.  Readings taken (two losses, both
# zero when every dimension is kept):
#   * query energy loss: the share of the projected query's squared norm on the
#     dimensions left out, 1 - sum_{j in S} q~_j^2 / sum_j q~_j^2;
#   * attention output loss: ||o_S - o|| / ||o||, o_S the output with scores on
#     the dimensions S only, o the standard attention output (all dimensions).
# The slicing baseline keeps dimensions 0 .. k-1 of the projected space (the
# largest singular values of the calibration).

def select_first_dims(k: int, d: int) -> np.ndarray:
    """The slicing baseline: the first k projected dimensions, whatever the query."""
    if not (1 <= k <= d):
        raise ValueError(f"need 1 <= k <= d, got k={k} d={d}")
    return np.arange(k)


def query_energy_loss(qt, S) -> float:
    """Share of the projected query's squared norm outside the kept dimensions S."""
    qt = np.asarray(qt, dtype=np.float64)
    total = float(np.dot(qt, qt))
    if total == 0.0:
        return 0.0
    kept = float(np.sum(qt[np.asarray(S)] ** 2))
    return 1.0 - kept / total


def attention_output_loss(qt, S, Kt, V, scale: float) -> float:
    """||o_S - o|| / ||o||: attention with scores on S against all dimensions (one head)."""
    d = np.shape(qt)[-1]
    s_full = sparse_scores(qt, np.arange(d), Kt, scale)
    s_S = sparse_scores(qt, S, Kt, scale)
    o = softmax(s_full)[0] @ np.asarray(V, dtype=np.float64)
    o_S = softmax(s_S)[0] @ np.asarray(V, dtype=np.float64)
    return float(np.linalg.norm(o_S - o) / np.linalg.norm(o))


def retention_losses(q, P, K, V, k: int, scale: float | None = None) -> dict:
    """Mean query-energy and attention-output losses of magnitude selection and
    of first-k slicing, over query heads q [H, d] attending to keys K [T, d]
    and values V [T, d] of one KV head with projection P [d, d]."""
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[-1]
    scale = default_scale(d) if scale is None else scale
    Kt = project(K, P)
    out = {"magnitude": {"energy": [], "output": []}, "slicing": {"energy": [], "output": []}}
    for h in range(q.shape[0]):
        qt = project(q[h], P)
        for name, S in (("magnitude", select_dims(qt, k)), ("slicing", select_first_dims(k, d))):
            out[name]["energy"].append(query_energy_loss(qt, S))
            out[name]["output"].append(attention_output_loss(qt, S, Kt, V, scale))
    return {name: {m: float(np.mean(v)) for m, v in r.items()} for name, r in out.items()}


# ----------------------------------------------------------------------------
# counts
# ----------------------------------------------------------------------------

def qk_macs(T: int, d: int, k: int | None = None) -> int:
    """Multiply-adds of the attention dot products of one query head over T tokens.

    Dense attention uses d per token; AQUA uses k per token (scores on the
    selected dimensions only).
    """
    return T * (d if k is None else k)


def breakeven_length(d: int, k: int, G: int) -> float:
    """Sequence length beyond which AQUA's decode multiply-adds undercut dense attention.

    The pages state that such a break-even point exists (abstract; edgentiq,
    Key Advantages) but print no formula.  Reading: per query head and decode
    step AQUA adds the query projection (d^2) and its share of the key
    projection (d^2 / G: one new key per KV head serves G query heads) and
    saves (d - k) per token, so T* = d^2 (1 + 1/G) / (d - k).  Counted in
    multiply-adds, not bytes.
    """
    if k >= d:
        return float("inf")
    return d * d * (1.0 + 1.0 / G) / (d - k)

