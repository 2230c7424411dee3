"""Pins of the fp64 speculative-verify oracle (oracle/spec.py), independent of its formulas.

* hand-derived inverse-CDF draws and worked acceptance tests (tests/golden);
* the defining property of the rule (the output has the target distribution),
  by Monte Carlo on a 5-token vocabulary with numpy's own sampler drawing the
  draft tokens. A dropped max(0, .), a swapped p and q, a reversed test or a
  draw from q instead of the residual each fail it;
* special cases: identical draft and target accept everything, a token the
  target forbids is never accepted or drawn, an out-of-range draft token is
  rejected, a zero residual falls back to the target row;
* invariance to a constant added to a row of logits.
"""
import os

import numpy as np
import pytest

from oracle import spec

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


def test_inverse_cdf_golden():
    n = 0
    for w, u, tok in _rows("spec_inverse_cdf.txt"):
        w = np.array([float(v) for v in w.split()])
        assert spec.inverse_cdf(w, float(u)) == int(tok), (w, u)
        n += 1
    assert n == 15


def _block_from_probs(p, q, d, r, G=1):
    lt = np.log(np.array([p] * (G + 1), dtype=np.float64)).astype(np.float32)
    ld = np.log(np.array([q] * G, dtype=np.float64)).astype(np.float32)
    return lt, ld, np.array([d] * G, dtype=np.int32), np.array([r] * G)


def test_acceptance_golden():
    p, q = [0.1, 0.2, 0.3, 0.4], [0.4, 0.3, 0.2, 0.1]
    n = 0
    for d, r, u, acc, tok in _rows("spec_accept.txt"):
        lt, ld, dd, rr = _block_from_probs(p, q, int(d), float(r))
        res = spec.verify_block(lt, ld, dd, rr, float(u))
        if int(acc):
            assert res["n"] == 1 and res["tokens"][0] == int(d)
        else:
            assert res["n"] == 0 and res["kind"] == "residual"
            assert res["tokens"] == [int(tok)]
        n += 1
    assert n == 8


def test_output_has_the_target_distribution():
    """Speculative sampling is lossless: every emitted position is distributed as
    the target's row for that position, whatever the draft distribution."""
    rng = np.random.default_rng(7)
    V, G, N = 5, 2, 40000
    lt = rng.normal(0, 1.2, size=(G + 1, V)).astype(np.float32)
    ld = rng.normal(0, 1.2, size=(G, V)).astype(np.float32)
    p = [spec.softmax(lt[i]) for i in range(G + 1)]
    q = [spec.softmax(ld[i]) for i in range(G)]
    counts = np.zeros((G + 1, V))
    n_acc0 = 0
    for _ in range(N):
        d = np.array([rng.choice(V, p=q[i]) for i in range(G)], dtype=np.int32)
        res = spec.verify_block(lt, ld, d, rng.random(G), rng.random())
        for pos, t in enumerate(res["tokens"]):
            counts[pos, t] += 1
        n_acc0 += res["n"] >= 1
    for pos in range(G + 1):
        m = counts[pos].sum()
        exp = m * p[pos]
        chi2 = ((counts[pos] - exp) ** 2 / exp).sum()
        assert chi2 < 30.0, (pos, chi2, counts[pos] / m, p[pos])  # df 4: p-value ~5e-6
    alpha = np.minimum(p[0], q[0]).sum()  # acceptance probability of position 0
    assert abs(n_acc0 / N - alpha) < 5 * np.sqrt(alpha * (1 - alpha) / N)


def test_identical_draft_accepts_every_token():
    rng = np.random.default_rng(3)
    V, G = 97, 8
    lt = rng.normal(0, 3, size=(G + 1, V)).astype(np.float32)
    for trial in range(20):
        d = rng.integers(0, V, size=G).astype(np.int32)
        res = spec.verify_block(lt, lt[:G].copy(), d, rng.random(G), rng.random())
        assert res["n"] == G and res["kind"] == "bonus"
        assert res["tokens"][:G] == d.tolist()


def test_forbidden_token_is_never_accepted_or_drawn():
    rng = np.random.default_rng(4)
    V, G = 50, 4
    lt = rng.normal(0, 1, size=(G + 1, V)).astype(np.float32)
    ld = rng.normal(0, 1, size=(G, V)).astype(np.float32)
    lt[0, 7] = -np.inf
    for trial in range(50):
        d = np.array([7] + list(rng.integers(0, V, size=G - 1)), dtype=np.int32)
        res = spec.verify_block(lt, ld, d, rng.random(G) * 0.999, rng.random())
        assert res["n"] == 0 and res["tokens"][0] != 7


def test_out_of_range_draft_token_is_rejected():
    rng = np.random.default_rng(5)
    V, G = 30, 3
    lt = rng.normal(0, 1, size=(G + 1, V)).astype(np.float32)
    d = np.array([1, V, 2], dtype=np.int32)
    res = spec.verify_block(lt, lt[:G].copy(), d, np.zeros(G), 0.5)
    assert res["n"] == 1 and res["tokens"][0] == 1
    # p == q at position 1: the residual is zero, so the draw falls back to p
    assert res["kind"] == "target"


def test_zero_residual_falls_back_to_target_row():
    lt = np.zeros((2, 4), dtype=np.float32)  # p = q = 1/4 each
    res = spec.verify_block(lt, lt[:1].copy(), np.array([0], dtype=np.int32), np.array([1.0]), 0.625)
    assert res["n"] == 0 and res["kind"] == "target" and res["tokens"] == [2]


def test_constant_shift_of_a_row_changes_nothing():
    rng = np.random.default_rng(6)
    V, G = 200, 8
    # multiples of 2^-10 in [-16, 16]: adding 64 is exact in fp32
    lt = (rng.integers(-16384, 16384, size=(G + 1, V)) / 1024.0).astype(np.float32)
    ld = (rng.integers(-16384, 16384, size=(G, V)) / 1024.0).astype(np.float32)
    d = rng.integers(0, V, size=G).astype(np.int32)
    r, u = rng.random(G), rng.random()
    a = spec.verify_block(lt, ld, d, r, u)
    b = spec.verify_block(lt + np.float32(64), ld - np.float32(64), d, r, u)
    assert a["n"] == b["n"] and a["tokens"] == b["tokens"]


def test_batch_pads_after_the_outputs():
    rng = np.random.default_rng(8)
    B, G, V = 6, 8, 40
    lt = rng.normal(0, 2, size=(B, G + 1, V)).astype(np.float32)
    ld = rng.normal(0, 2, size=(B, G, V)).astype(np.float32)
    d = rng.integers(0, V, size=(B, G)).astype(np.int32)
    n, toks = spec.verify(lt, ld, d, rng.random((B, G)), rng.random(B))
    for b in range(B):
        assert (toks[b, :n[b]] == d[b, :n[b]]).all()
        assert 0 <= toks[b, n[b]] < V
        assert (toks[b, n[b] + 1:] == -1).all()


def test_unpinned_helpers():
    assert spec.decision_unpinned(0.5, 0.25, 0.5, 1000)
    assert not spec.decision_unpinned(0.49, 0.25, 0.5, 1000)
    w = np.array([1.0, 1.0, 2.0, 4.0])
    assert spec.sample_unpinned(w, 0.25, 4, "bonus")[0]  # u*S lands on C_1
    assert not spec.sample_unpinned(w, 0.3, 4, "bonus")[0]
    pinned, cands = spec.sample_unpinned(w, 0.25, 4, "bonus")
    assert {1, 2} <= cands


@pytest.mark.parametrize("name", ["verify_tiny_v1000_g8"])
def test_synthetic_blocks_accept_most_drafts(name):
    """The input recipe's blocks accept most drafts: with the draft close to the
    target, about 95% per position."""
    from synth.spec import VERIFY_WORKLOADS, verify_inputs
    w = VERIFY_WORKLOADS[name].with_blocks(16)
    inp = verify_inputs(w, seed=0)
    n, toks = spec.verify(inp["lt"], inp["ld"], inp["d"], inp["r"], inp["u"])
    assert n.mean() > 4.0
    assert ((toks >= -1) & (toks < w.vocab)).all()
