"""fp64 speculative-verify acceptance step (rejection sampling over one verify block).

Test infrastructure: only tests/, __graft_entry__.smoke() and bench.py's CPU
legs use this module. The product path never calls it.

What it follows. A draft model proposes a block of tokens and the main model
verifies them. Rejection sampling in the verify stage keeps the output
distribution that of standard decoding (bjdmk news on MiMo-V2.5-Pro-UltraSpeed,
section "极致协同，通向千速之路"; yifor blog "Xiaomi MiMo and TileRT Push a
1-Trillion-Parameter Model Past 1000 Tokens Per Second on Commodity GPUs",
item 2 on DFlash speculative decoding). The block is 8 draft tokens (bjdmk
news, same section). The draft fills the whole block in one pass, so every
position has its own draft distribution.

The pages name the rule but do not spell it out. The plainest reading is the
standard speculative-sampling acceptance rule, whose output has exactly the
target model's distribution:

* p_i = softmax(target logits of position i), i = 0 .. G (row G scores the
  position after the last draft token); q_i = softmax(draft logits of
  position i), i = 0 .. G-1; softmax(l)_j = exp(l_j - max l) / sum_k exp(l_k - max l);
* for i = 0, 1, ...: draft token d_i is accepted when r_i * q_i(d_i) < p_i(d_i).
  This is r_i < min(1, p_i(d_i) / q_i(d_i)), with r_i uniform in [0, 1), and
  it also covers q_i(d_i) = 0. A d_i outside [0, V) is rejected;
* at the first rejection, position n = i, one token is drawn from the residual
  weights max(0, p_n - q_n). If those weights sum to zero (possible only in
  rounding), the token is drawn from p_n. Nothing after position n is looked at;
* if all G drafts are accepted, n = G and one token is drawn from p_G;
* drawing from weights w with uniform u in [0, 1): the smallest j whose
  cumulative sum C_j = w_0 + ... + w_j exceeds u * C_{V-1} (inverse CDF).
  A token with w_j = 0 is never drawn;
* output: n, and the n + 1 tokens d_0 .. d_{n-1}, t_n.

Temperature is not a parameter: a caller folds it into the logits. All
arithmetic is fp64 on the fp32 logits, sums in index order.
"""
from __future__ import annotations

import numpy as np

U64 = 2.0 ** -53  # unit roundoff of fp64


def softmax(l: np.ndarray) -> np.ndarray:
    """exp(l - max l) / sum exp(l - max l) in fp64, the sum in index order."""
    l = np.asarray(l, dtype=np.float64)
    e = np.exp(l - l.max())
    return e / np.cumsum(e)[-1]


def inverse_cdf(w: np.ndarray, u: float) -> int:
    """Smallest j with w_0 + ... + w_j > u * (w_0 + ... + w_{V-1}) (sums in index order).

    When rounding leaves no such j (u * S == S), the last j with w_j > 0."""
    c = np.cumsum(np.asarray(w, dtype=np.float64))
    j = int(np.searchsorted(c, u * c[-1], side="right"))
    if j >= len(c):
        j = int(np.flatnonzero(np.asarray(w) > 0)[-1])
    return j


def accepts(r: float, p_d: float, q_d: float) -> bool:
    """The acceptance test of one draft token: r * q(d) < p(d)."""
    return r * q_d < p_d


def verify_block(lt: np.ndarray, ld: np.ndarray, d: np.ndarray, r: np.ndarray, u: float) -> dict:
    """One verify block: lt [G+1][V], ld [G][V], d [G], r [G], u.

    Returns n (accepted drafts), the n + 1 output tokens, the sampled
    distribution's weights and the row it came from ("residual", "target"
    or "bonus"), and the acceptance ratios that were tested."""
    G, V = ld.shape[0], lt.shape[1]
    tested = []
    for i in range(G):
        p, q = softmax(lt[i]), softmax(ld[i])
        di = int(d[i])
        if 0 <= di < V:
            tested.append((r[i], p[di], q[di]))
            if accepts(r[i], p[di], q[di]):
                continue
        w = np.maximum(p - q, 0.0)
        kind = "residual"
        if np.cumsum(w)[-1] == 0.0:
            w, kind = p, "target"
        t = inverse_cdf(w, u)
        return {"n": i, "tokens": [int(x) for x in d[:i]] + [t], "weights": w, "kind": kind,
                "tested": tested}
    p = softmax(lt[G])
    t = inverse_cdf(p, u)
    return {"n": G, "tokens": [int(x) for x in d] + [t], "weights": p, "kind": "bonus", "tested": tested}


def verify(lt: np.ndarray, ld: np.ndarray, d: np.ndarray, r: np.ndarray, u: np.ndarray):
    """B verify blocks: returns n [B] and tokens [B][G+1] (-1 after the n + 1 outputs)."""
    B, G = d.shape
    n = np.empty(B, dtype=np.int32)
    toks = np.full((B, G + 1), -1, dtype=np.int32)
    for b in range(B):
        res = verify_block(lt[b], ld[b], d[b], r[b], float(u[b]))
        n[b] = res["n"]
        toks[b, :res["n"] + 1] = res["tokens"]
    return n, toks


# ---- rounding bounds, for comparing a GPU result taken in another summation order ----

def prob_rel_bound(V: int) -> float:
    """Bound on the relative error of a softmax probability computed in fp64 by
    any summation order. It covers V terms summed, one exp of at most 2 ulp, one
    more exp per partial sum rescaled to a common maximum, and the division.
    Scaled by 4 for margin."""
    return 4.0 * (V + 8) * U64


def decision_unpinned(r: float, p_d: float, q_d: float, V: int) -> bool:
    """True when r*q(d) and p(d) are so close that another fp64 evaluation may
    decide the other way."""
    e = prob_rel_bound(V)
    return abs(r * q_d - p_d) <= e * (p_d + r * q_d) + 1e-300


def sample_unpinned(w: np.ndarray, u: float, V: int, kind: str) -> tuple[bool, set]:
    """Whether the inverse-CDF draw from w at u is pinned, and, if not, the set of
    tokens another fp64 evaluation could return.

    Every cumulative sum C_j computed in another order differs by at most
    bound = e * (sum of the terms that make up w). For residual weights each
    term is within e of the two probabilities it subtracts; for a target or
    bonus row it is within e of p_j. A draw is unpinned when u * S lies within
    2 * bound of a boundary C_j. The candidates are then the tokens with
    positive weight on either side of every such boundary."""
    w = np.asarray(w, dtype=np.float64)
    c = np.cumsum(w)
    S = c[-1]
    e = prob_rel_bound(V)
    bound = e * (2.0 if kind == "residual" else 1.0) * (1.0 + S) + 4.0 * V * U64 * S
    t = u * S
    near = np.flatnonzero(np.abs(c - t) <= 2.0 * bound + 2.0 * U64 * S)
    if near.size == 0:
        return False, {inverse_cdf(w, u)}
    pos = np.flatnonzero(w > 0)
    cands = {inverse_cdf(w, u)}
    for j in near:
        k = np.searchsorted(pos, j, side="left")
        for kk in (k - 1, k, k + 1):
            if 0 <= kk < len(pos):
                cands.add(int(pos[kk]))
    return True, cands
