"""Plain fp64 CPU oracle for the DoSA certified indexer Top-K.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The CUDA library never calls it, and it shares no code with the CUDA
path (no kernels, headers, tables or helpers).

Sources (all web pages on DoSA):
  [DPC]  "DOSA: Dots Sparse Attention", Daily Paper Cast transcript.
         Sections: Introduction, Method, Experiments and Results, Related Work.
  [ZICQ] "arXiv Releases DoSA: Revolutionizing Sparse Attention for Enhanced
         Indexing Efficiency and Inference Speed", Technical Mechanism Analysis.
  [PICX] "Xiaohongshu DoSA sparse attention cuts TTFT by up to 48% via score
         bounds", sections 01-03 of the quoted article.

What the method computes.  The pages state that DoSA keeps the original scoring
function and returns exactly the Top-K the dense indexer returns ([PICX] 02,
[ZICQ] point 2: the token selection is exact; [DPC] Introduction: a rejected
key could never have been among the Top-K).  So the dense oracle below is the plain
definition: decode the stored inputs exactly, score every visible key in fp64,
sort, take K.  The certificate half follows the steps of [DPC] Method in order
(seed threshold, three bound stages, tile-by-tile refinement); the pages print
no formula, so every formula here is the plainest construction consistent with
the wording; the docstring of each function states the reading it takes.

Parity status of each function (pins live in tests/test_oracle_*.py):
  decode_bf16, decode_e4m3 ...... pinned (format definitions, hand values, torch)
  indexer_scores ................ pinned (brute-force loops, integer closed forms)
  select_topk ................... pinned (repeated argmax, sorted() on tuples)
  nnls_retained ................. pinned (grid search, KKT conditions)
  certificate_setup/upper_bound . pinned (UB >= I invariant, closed-form reductions)
  certified_topk_row ............ pinned (equals dense selection; tau <= K-th;
                                  ideal_rejected in the closed form UB = I)
  ranked_topk_row ............... pinned (equals dense selection; every rejected
                                  key scores below the K-th; rejected <= ideal)
  key_block_stats/block_upper_bound  pinned (bound >= every key's UB in the
                                  block, single-key blocks reduce to UB)
  prune rates ................... parity unpinned against the pages (their ~97 %
                                  is measured on trained indexers); pinned only
                                  by the ideal-rate upper limit.
"""
from __future__ import annotations

import itertools
import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "decode_bf16", "decode_e4m3", "dequantize", "indexer_scores", "select_topk",
    "dense_topk", "nnls_retained", "Certificate", "certificate_setup", "upper_bound",
    "soundness_margin", "seed_mask", "certified_topk_row", "certified_topk",
    "key_mean", "key_block_stats", "block_upper_bound", "ranked_topk_row",
]

# ----------------------------------------------------------------------------
# Exact decoding of the stored number formats.
# ----------------------------------------------------------------------------


def decode_bf16(codes: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64, from the format: 1 sign bit, 8 exponent
    bits (bias 127), 7 fraction bits; exponent 0 is subnormal.  Inf/NaN codes
    are rejected (the indexer inputs are finite)."""
    c = np.asarray(codes).astype(np.int64)
    sign = np.where((c >> 15) & 1, -1.0, 1.0)
    e = (c >> 7) & 0xFF
    f = (c & 0x7F).astype(np.float64)
    if np.any(e == 0xFF):
        raise ValueError("bf16 input holds Inf or NaN")
    normal = np.ldexp(1.0 + f / 128.0, (e - 127).astype(np.int64))
    sub = np.ldexp(f / 128.0, -126)
    return sign * np.where(e == 0, sub, normal)


def _e4m3_table() -> np.ndarray:
    """The 256 values of OCP FP8 E4M3 (the 'fn' variant: no infinities).
    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.  Exponent 0 is
    subnormal (m/8 * 2^-6).  Only S.1111.111 is NaN; S.1111.110 = 448 is the
    largest finite value."""
    table = np.empty(256, np.float64)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            table[code] = np.nan
        elif e == 0:
            table[code] = s * (m / 8.0) * 2.0 ** -6
        else:
            table[code] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return table


_E4M3 = _e4m3_table()


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """e4m3 bit patterns -> float64 through the table above.  NaN codes are
    rejected."""
    v = _E4M3[np.asarray(codes).astype(np.int64)]
    if np.any(np.isnan(v)):
        raise ValueError("e4m3 input holds NaN")
    return v


def dequantize(codes: np.ndarray, scale: np.ndarray | None, dtype: str) -> np.ndarray:
    """Stored value -> real value.  bf16: the value itself.  fp8: one fp32
    scale per token multiplies the decoded code (the per-token scale of the
    128K/1M workloads), applied in fp64 over the leading axis."""
    if dtype == "bf16":
        return decode_bf16(codes)
    if dtype == "fp8":
        v = decode_e4m3(codes)
        s = np.asarray(scale, np.float64).reshape((-1,) + (1,) * (v.ndim - 1))
        return v * s
    raise ValueError(f"unknown dtype {dtype!r}")


# ----------------------------------------------------------------------------
# Dense indexer: the definition.
# ----------------------------------------------------------------------------


def indexer_scores(q_t: np.ndarray, w_t: np.ndarray, k: np.ndarray) -> np.ndarray:
    """I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s]) for every row s of ``k``.

    The signed multi-head indexer score that DoSA keeps unchanged ([DPC] Method,
    problem formulation: one query with several indexer heads, each with its own
    query vector and weight, scored against shared keys; [PICX] 01: the indexer
    scores candidates and keeps the K highest).  q_t: [H, d], w_t: [H], k: [n, d],
    all float64.  Returns [n] float64."""
    x = k @ q_t.T                        # [n, H]: one dot product per (key, head)
    return np.maximum(x, 0.0) @ w_t      # ReLU, then the weighted head sum


def select_topk(scores: np.ndarray, K: int) -> np.ndarray:
    """Indices of the K largest scores, ties to the smaller index, returned in
    ascending index order and padded with -1 when fewer than K keys exist.

    The dense baseline scores every key and then takes the Top-K ([DPC]
    Experiments, baselines).  Tie rule: smaller key index wins."""
    n = int(scores.shape[0])
    order = np.lexsort((np.arange(n), -scores))     # -score ascending, then index
    chosen = np.sort(order[: min(K, n)])
    out = np.full(K, -1, np.int64)
    out[: chosen.shape[0]] = chosen
    return out


def dense_topk(q: np.ndarray, w: np.ndarray, k: np.ndarray, positions: np.ndarray,
               K: int, rows=None) -> np.ndarray:
    """Dense Top-K for every query row (or the listed ``rows``) of one sequence.

    q: [T, H, d] real values, w: [T, H], k: [S, d] real values, positions: [T]
    (query row i sees keys 0..positions[i], causal s <= t).  Returns [len(rows), K]."""
    rows = range(q.shape[0]) if rows is None else rows
    out = []
    for t in rows:
        p = int(positions[t])
        out.append(select_topk(indexer_scores(q[t], w[t].astype(np.float64), k[: p + 1]), K))
    return np.stack(out) if out else np.zeros((0, K), np.int64)


# ----------------------------------------------------------------------------
# Certificate ([DPC] Method: three stages; [ZICQ] Technical Mechanism Analysis).
# ----------------------------------------------------------------------------


def nnls_retained(Q_R: np.ndarray, v: np.ndarray) -> np.ndarray:
    """alpha = argmin_{alpha >= 0} || v - alpha @ Q_R ||  (Q_R: [r, d], v: [d]).

    The pages keep some positive-weight heads and project the others onto
    them so that the projection residual is as small as possible ([DPC]
    Method), with coefficients that are nonnegative ([DPC] Conclusion;
    [ZICQ] point 2).  Solved exactly for
    r <= 4 by trying every support: the NNLS optimum is the unconstrained
    least-squares solution on its own support, so the best feasible candidate
    over all supports is the optimum.  For more retained heads (the head-budget
    study) scipy's NNLS routine (Lawson and Hanson's active-set method) serves
    as the step."""
    r = Q_R.shape[0]
    if r > 4:
        from scipy.optimize import nnls
        alpha, _ = nnls(Q_R.T, v)
        return alpha
    best_alpha = np.zeros(r)
    best_res = float(v @ v)
    for size in range(1, r + 1):
        for support in itertools.combinations(range(r), size):
            B = Q_R[list(support)]                       # [size, d]
            a, *_ = np.linalg.lstsq(B.T, v, rcond=None)  # unconstrained LS on the support
            if np.all(a >= 0.0):
                res_vec = v - a @ B
                res = float(res_vec @ res_vec)
                if res < best_res:
                    best_res = res
                    best_alpha = np.zeros(r)
                    best_alpha[list(support)] = a
    return best_alpha


@dataclass
class Certificate:
    """Per-query certificate: UB(k) = sum_j omega_j ReLU(q_j.k) + beta ||k||
    - sum_g ReLU(u_g.k)."""
    retained: np.ndarray                 # R: indices of the exactly evaluated heads
    omega: np.ndarray                    # [|R|] folded weights of the retained heads
    beta: float                          # joint residual coefficient (times ||k||)
    beta_sum: float                      # the per-head Cauchy-Schwarz sum (for reports)
    beta_joint: float                    # the joint (spectral) bound (for reports)
    groups: list = field(default_factory=list)   # negative supports A_g (head indices)
    u: np.ndarray = None                 # [G, d] aggregated negative directions


def certificate_setup(q_t: np.ndarray, w_t: np.ndarray, k_bar: np.ndarray,
                      r: int, G: int) -> Certificate:
    """Build the certificate of one query (real-valued q_t [H, d], w_t [H]).

    Stage 1, positive heads ([DPC] Method: the positive heads left out are
    bounded from above; [ZICQ] 2: nonnegative projections and one joint bound
    on the residuals cap what the positive heads can add):
      P = {h : w_h > 0}; R = the r heads of P with the largest w_h ||q_h||
      (ties to the smaller head).  For each omitted h in O = P \\ R,
      alpha_h = NNLS projection onto the retained heads, rho_h its residual.
      ReLU is positively homogeneous and subadditive, and alpha >= 0, so
        ReLU(q_h.k) <= sum_j alpha_hj ReLU(q_j.k) + |rho_h.k|.
      The retained heads' dot products are computed once and reused ([DPC]
      Method):
        omega_j = w_j + sum_{h in O} w_h alpha_hj.
      Joint residual bound: sum_h w_h |rho_h.k| <= beta ||k|| with
        beta = min( sum_h w_h ||rho_h|| ,  sqrt( W_O * lambda_max(M) ) ),
        W_O = sum_{h in O} w_h,  M = sum_{h in O} w_h rho_h rho_h^T
      (the second is Cauchy-Schwarz with weights w_h, then the spectral norm:
      it bounds all residual heads jointly).
    Stage 2, negative heads ([DPC] Method: the negative heads are summed over
    supports chosen from which heads are active; [ZICQ] 2: that aggregate
    bounds how much the negative heads can subtract):
      for a >= 0, sum_{h in A} a_h ReLU(x_h) >= ReLU(sum_{h in A} a_h x_h).
      N = {h : w_h < 0}.  A_1 = {h in N : q_h.k_bar > 0} (heads active on the
      mean key), A_2 = N \\ A_1 when G >= 2.  u_g = sum_{h in A_g} |w_h| q_h.
    Heads with w_h = 0 contribute nothing and are dropped."""
    H = q_t.shape[0]
    w = w_t.astype(np.float64)
    qn = np.linalg.norm(q_t, axis=1)
    P = [h for h in range(H) if w[h] > 0.0]
    N = [h for h in range(H) if w[h] < 0.0]
    # top-r of P by w_h ||q_h||, ties to the smaller head index
    ranked = sorted(P, key=lambda h: (-(w[h] * qn[h]), h))
    R = np.array(sorted(ranked[: min(r, len(P))]), np.int64)
    O = [h for h in P if h not in set(R.tolist())]

    omega = w[R].copy() if R.size else np.zeros(0)
    rhos = []
    for h in O:
        alpha = nnls_retained(q_t[R], q_t[h]) if R.size else np.zeros(0)
        omega = omega + w[h] * alpha
        rhos.append(q_t[h] - (alpha @ q_t[R] if R.size else 0.0))
    if O:
        rho = np.array(rhos)                              # [|O|, d]
        wO = w[O]
        beta_sum = float(np.sum(wO * np.linalg.norm(rho, axis=1)))
        Ws = np.sqrt(wO)[:, None] * rho
        lam = float(np.linalg.eigvalsh(Ws @ Ws.T)[-1])    # lambda_max(M) via the Gram matrix
        beta_joint = math.sqrt(float(wO.sum()) * max(lam, 0.0))
        beta = min(beta_sum, beta_joint)
    else:
        beta_sum = beta_joint = beta = 0.0

    groups = []
    if G >= 1 and N:
        act = q_t[N] @ k_bar
        A1 = [h for h, a in zip(N, act) if a > 0.0]
        groups.append(np.array(A1, np.int64))
        if G >= 2:
            groups.append(np.array([h for h in N if h not in set(A1)], np.int64))
    d = q_t.shape[1]
    u = np.zeros((len(groups), d))
    for g, A in enumerate(groups):
        if A.size:
            u[g] = (np.abs(w[A])[:, None] * q_t[A]).sum(axis=0)
    return Certificate(R, omega, beta, beta_sum, beta_joint, groups, u)


def upper_bound(cert: Certificate, q_t: np.ndarray, k: np.ndarray) -> np.ndarray:
    """Stage 3, the combined bound ([DPC] Method: one certificate per key adds
    the retained heads' exact terms and the bounds of the other heads):
      UB(s) = sum_j omega_j ReLU(q_j.k_s) + beta ||k_s|| - sum_g ReLU(u_g.k_s).
    k: [n, d] real values.  UB(s) >= I(t,s) for every key (tests pin this)."""
    ub = cert.beta * np.linalg.norm(k, axis=1)
    if cert.retained.size:
        ub = ub + np.maximum(k @ q_t[cert.retained].T, 0.0) @ cert.omega
    for g in range(cert.u.shape[0]):
        ub = ub - np.maximum(k @ cert.u[g], 0.0)
    return ub


def key_block_stats(k_block: np.ndarray) -> tuple[np.ndarray, float, float]:
    """A block of keys summarised by a ball: its center (the mean key), the
    radius max_s ||k_s - center|| and the largest key norm."""
    k_block = np.asarray(k_block, np.float64)
    c = k_block.mean(axis=0)
    r = float(np.max(np.linalg.norm(k_block - c, axis=1)))
    n = float(np.max(np.linalg.norm(k_block, axis=1)))
    return c, r, n


def block_upper_bound(cert: Certificate, q_t: np.ndarray, center: np.ndarray, radius: float,
                      max_norm: float) -> float:
    """One bound for every key of a block ("DOSA: Dots Sparse Attention",
    Daily Paper Cast transcript, future work: extending the certificate from
    single keys to key blocks, cutting scoring and key-access costs).  Every key of
    the block is k = center + e with ||e|| <= radius, so for any vector v
    v.k lies in [v.center - ||v|| radius, v.center + ||v|| radius].  ReLU is
    nondecreasing, omega_j >= 0 and ||k|| <= max_norm, hence each term of the
    per-key bound (upper_bound) is at most its block counterpart:
      UB_B = sum_j omega_j ReLU(q_j.c + ||q_j|| r) + beta max_norm
             - sum_g ReLU(u_g.c - ||u_g|| r)  >=  UB(s)  for every s in B."""
    ub = cert.beta * max_norm
    for j, h in enumerate(cert.retained):
        ub += cert.omega[j] * max(float(q_t[h] @ center) + float(np.linalg.norm(q_t[h])) * radius,
                                  0.0)
    for g in range(cert.u.shape[0]):
        ub -= max(float(cert.u[g] @ center) - float(np.linalg.norm(cert.u[g])) * radius, 0.0)
    return ub


def soundness_margin(q_t: np.ndarray, w_t: np.ndarray, k: np.ndarray,
                     margin_log2: int) -> np.ndarray:
    """delta(t,s) = 2^margin_log2 * (sum_h |w_h| ||q_h||) * ||k_s||.

    The pages are silent on rounding.  A GPU evaluates the bound and the score
    in fp32 with different arithmetic, so a candidate is rejected only when
    UB + delta < tau.  delta dominates the fp32 error of both sides."""
    c = float(np.sum(np.abs(w_t.astype(np.float64)) * np.linalg.norm(q_t, axis=1)))
    return math.ldexp(c, margin_log2) * np.linalg.norm(k, axis=1)


def seed_mask(p: int, seed_first: int, seed_last: int) -> np.ndarray:
    """Seed subset of the visible keys 0..p: the first ``seed_first`` keys and the
    last ``seed_last`` keys ending at p ([DPC] Method: the threshold starts as
    the K-th largest exact score over a subset of the visible keys)."""
    s = np.arange(p + 1)
    return (s < seed_first) | (s > p - seed_last)


def key_mean(k: np.ndarray) -> np.ndarray:
    """Mean key of a sequence: the direction on which head activation is read
    when choosing the negative support."""
    return k.mean(axis=0) if k.shape[0] else np.zeros(k.shape[1])


def _kth_largest(values: np.ndarray, K: int) -> float:
    if values.shape[0] < K:
        return -math.inf
    return float(np.partition(values, values.shape[0] - K)[values.shape[0] - K])


def certified_topk_row(q_t, w_t, k_vis, K, *, k_bar, r=4, G=2, seed_first=64,
                       seed_last=512, margin_log2=-12, tile=128) -> dict:
    """One query through the certified pipeline ([DPC] Method, candidate
    refinement: screening dot products, bound evaluation, pruning and score
    compaction, repeated for every tile of visible keys).

      1. Exact scores on the seed subset; tau = their K-th largest (-inf while
         fewer than K exact scores exist).
      2. The remaining keys, in tiles of ``tile`` keys aligned to absolute key
         positions, from the diagonal downwards: a key is rejected when
         UB + delta < tau; every survivor is scored with all heads.  After
         each tile tau is raised to the K-th largest exact score so far (any
         such K-th is a lower bound on the true K-th).
      3. Top-K over the exactly scored keys.

    k_vis: [p+1, d] real values of the visible keys.  Returns the selection and
    the counts used for the prune rate ([DPC] Experiments: the share of
    query-key pairs that screening removes)."""
    n = k_vis.shape[0]
    p = n - 1
    w64 = w_t.astype(np.float64)
    cert = certificate_setup(q_t, w64, k_bar, r, G)
    exact = np.full(n, np.nan)
    seeds = seed_mask(p, seed_first, seed_last)
    exact[seeds] = indexer_scores(q_t, w64, k_vis[seeds])
    tau0 = _kth_largest(exact[seeds], K)
    tau = tau0
    ub = upper_bound(cert, q_t, k_vis)
    delta = soundness_margin(q_t, w64, k_vis, margin_log2)
    rejected = np.zeros(n, bool)
    rest = np.nonzero(~seeds)[0]
    if rest.size:
        for tile_start in range((int(rest.max()) // tile) * tile, -1, -tile):
            sel = rest[(rest >= tile_start) & (rest < tile_start + tile)]
            if sel.size == 0:
                continue
            rej = ub[sel] + delta[sel] < tau
            rejected[sel[rej]] = True
            keep = sel[~rej]
            if keep.size:
                exact[keep] = indexer_scores(q_t, w64, k_vis[keep])
            tau = max(tau, _kth_largest(exact[~np.isnan(exact)], K))
    scored = np.nonzero(~np.isnan(exact))[0]
    vals = exact[scored]
    order = np.lexsort((scored, -vals))
    chosen = np.sort(scored[order[: min(K, scored.size)]])
    idx = np.full(K, -1, np.int64)
    idx[: chosen.size] = chosen
    # ideal screening: tau equal to the true K-th score
    full = indexer_scores(q_t, w64, k_vis)
    vK = _kth_largest(full, K)
    ideal_rej = (~seeds) & (ub + delta < vK)
    return {
        "idx": idx, "tau0": tau0, "tau_final": tau, "v_K": vK,
        "visible": n, "seed": int(seeds.sum()), "screened": int((~seeds).sum()),
        "rejected": int(rejected.sum()), "ideal_rejected": int(ideal_rej.sum()),
        "cert": cert, "ub": ub, "delta": delta, "scores": full,
    }


def certified_topk(q, w, k, positions, K, rows=None, **kw) -> tuple[np.ndarray, dict]:
    """certified_topk_row over several rows of one sequence; returns the
    selections and summed counts (visible, seed, screened, rejected, ideal)."""
    rows = range(q.shape[0]) if rows is None else rows
    k_bar = kw.pop("k_bar", None)
    if k_bar is None:
        k_bar = key_mean(k)
    out, tot = [], {"visible": 0, "seed": 0, "screened": 0, "rejected": 0, "ideal_rejected": 0}
    for t in rows:
        p = int(positions[t])
        res = certified_topk_row(q[t], w[t], k[: p + 1], K, k_bar=k_bar, **kw)
        out.append(res["idx"])
        for key in tot:
            tot[key] += res[key]
    return (np.stack(out) if out else np.zeros((0, K), np.int64)), tot


def ranked_topk_row(q_t, w_t, k_vis, K, *, k_bar, warm_tiles, r=4, G=2, seed_first=64,
                    seed_last=512, margin_log2=-12, tile=128, spread=1.5, growth=8) -> dict:
    """One query through the certified pipeline with a ranked threshold
    schedule.  The pages fix what is computed (seed threshold, certificate,
    rejection, all-head scoring of the survivors; [DPC] Method, candidate
    refinement) but not in which order the keys are screened; this reading
    screens every remaining key against an estimate of the threshold and
    checks the estimate afterwards:

      1. Warm-up: key tile 0 and the warm_tiles - 1 tiles ending at the
         diagonal are scored exactly (n_e keys).  The seed subset is scored
         exactly wherever it lies.
      2. Estimates U_1 > U_2 > ...: U_j = the m_j-th largest warm-up score,
         m_1 = ceil(spread * K * n_e / n), m_{j+1} = growth * m_j, clamped to
         [1, K].  U_1 estimates a score a little below the K-th (the warm-up
         keys as a sample of the n visible keys); the last, m = K, is the
         warm-up's own K-th largest score, a sound threshold.
      3. Pass 1: every other key is a survivor when v = UB + delta >= U_1 and
         is scored exactly.
      4. After pass j, tau = the K-th largest exact score so far (a lower bound
         on the true K-th, as any subset's K-th is).  If a key not scored yet
         has v >= tau, pass j + 1 scores exactly the keys with
         max(tau, U_{j+1}) <= v < (pass j's lower limit).  Once U_{j+1} <= tau
         that pass leaves no key with v >= tau unscored, so the schedule ends.
      5. Top-K over the exactly scored keys.
    Every rejected key has I <= v < tau <= v_K, so the selection is the dense
    one.  Returns the selection and the counts of the prune rate."""
    n = k_vis.shape[0]
    p = n - 1
    w64 = w_t.astype(np.float64)
    cert = certificate_setup(q_t, w64, k_bar, r, G)
    full = indexer_scores(q_t, w64, k_vis)
    v = upper_bound(cert, q_t, k_vis) + soundness_margin(q_t, w64, k_vis, margin_log2)
    keys = np.arange(n)
    n_tiles = p // tile + 1
    first_diag = max(1, n_tiles - warm_tiles + 1)
    warm = (keys < tile) | (keys >= first_diag * tile)
    seeds = seed_mask(p, seed_first, seed_last)
    n_e = int(warm.sum())
    m = min(K, max(1, int(math.ceil(spread * K * n_e / n))))
    estimates = [_kth_largest(full[warm], m)]
    ms = [m]
    while ms[-1] < K:
        ms.append(min(K, ms[-1] * growth))
        estimates.append(_kth_largest(full[warm], ms[-1]))
    screened = ~warm & ~seeds
    lower = estimates[0]
    exact = warm | seeds | (screened & (v >= lower))
    survived_1 = int((screened & exact).sum())
    passes = 1
    while True:
        tau = _kth_largest(full[exact], K)
        if not np.any(v[screened & ~exact] >= tau):
            break
        nxt = estimates[passes] if passes < len(estimates) else -math.inf
        new_lower = max(tau, nxt)
        exact = exact | (screened & (v >= new_lower) & (v < lower))
        lower = new_lower
        passes += 1
    scored = np.nonzero(exact)[0]
    vals = full[scored]
    order = np.lexsort((scored, -vals))
    chosen = np.sort(scored[order[: min(K, scored.size)]])
    idx = np.full(K, -1, np.int64)
    idx[: chosen.size] = chosen
    vK = _kth_largest(full, K)
    return {
        "idx": idx, "u_hat": estimates[0], "estimates": estimates, "m": ms[0], "n_warm": n_e,
        "tau": tau, "passes": passes, "v_K": vK, "visible": n, "seed": int(seeds.sum()),
        "screened": int(screened.sum()), "survived_1": survived_1,
        "rejected": int((screened & ~exact).sum()),
        "ideal_rejected": int((screened & (v < vK)).sum()),
        "exact": int(exact.sum()), "scores": full, "bound": v, "exact_mask": exact,
    }
