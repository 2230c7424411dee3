"""The speculative-verify acceptance kernel (spec_verify) against the fp64 oracle.

Compared per block: the number of accepted drafts, every output token and the
-1 padding. Both sides decide in fp64. Only a decision or a draw that the
oracle's rounding bound marks as unpinned may differ: another summation order
can move a value across its threshold there. Such cases are counted, and the
GPU's token must still be one the bound allows.
"""
import numpy as np
import pytest

from synth.spec import VERIFY_WORKLOADS, VerifyWorkload, verify_inputs
from tests.gpu_helpers import check_verify as check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from tests.gpu_helpers import mx as load
    return load()


def _dev(inp):
    import torch
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in inp.items()}


def _run(mx, inp, sv=None):
    B, G = inp["d"].shape
    V = inp["lt"].shape[2]
    sv = sv or mx.SpecVerify(B, G, V)
    t = _dev(inp)
    n, toks = sv(t["lt"], t["ld"], t["d"], t["r"], t["u"])
    sv.status()
    return n.cpu().numpy(), toks.cpu().numpy()


@pytest.mark.parametrize("V,G,B", [(1000, 8, 4), (4099, 8, 3), (512, 8, 2), (513, 8, 2), (33, 8, 5),
                                   (1, 8, 2), (2000, 0, 3), (3000, 1, 4), (1500, 16, 2), (16384, 8, 7)])
def test_matches_oracle(mx, V, G, B):
    w = VerifyWorkload("t", V, G, B)
    inp = verify_inputs(w, seed=V + G)
    n, toks = _run(mx, inp)
    assert check(inp, n, toks) == 0


@pytest.mark.parametrize("name", ["verify_b1_v152064_g8", "verify_b64_v152064_g8"])
def test_full_size_workloads_match_oracle(mx, name):
    w = VERIFY_WORKLOADS[name]
    inp = verify_inputs(w, seed=0)
    n, toks = _run(mx, inp)
    assert check(inp, n, toks) == 0


def test_residual_draws_over_many_seeds(mx):
    """A far draft (every block rejects early), so most blocks draw from the residual."""
    w = VerifyWorkload("far", 20000, 8, 32, draft_noise=3.0)
    loose = 0
    for seed in range(4):
        inp = verify_inputs(w, seed=seed)
        n, toks = _run(mx, inp)
        assert (n < 8).mean() > 0.5
        loose += check(inp, n, toks)
    assert loose <= 1


def test_identical_draft_accepts_all_and_draws_bonus(mx):
    w = VerifyWorkload("same", 7000, 8, 6)
    inp = verify_inputs(w, seed=5)
    inp["ld"] = np.ascontiguousarray(inp["lt"][:, :8])
    n, toks = _run(mx, inp)
    assert (n == 8).all()
    assert check(inp, n, toks) == 0


def test_edge_tokens(mx):
    """Masked target token, out-of-range drafts, r = 0 and uniform rows (ties everywhere)."""
    w = VerifyWorkload("edge", 3000, 4, 5)
    inp = verify_inputs(w, seed=9)
    inp["lt"][0, 0, inp["d"][0, 0]] = -np.inf      # block 0: first draft forbidden
    inp["d"][1, 1] = 3000                           # block 1: second draft out of range
    inp["d"][2, 0] = -5                             # block 2: first draft negative
    inp["r"][3] = 0.0                               # block 3: accept whatever p > 0
    inp["lt"][4] = 0.0                              # block 4: uniform target rows
    inp["ld"][4] = 0.0
    inp["u"][4] = 0.5
    n, toks = _run(mx, inp)
    assert n[0] == 0 and toks[0, 0] != inp["d"][0, 0]
    assert n[1] <= 1 and n[2] == 0
    assert n[3] == 4
    assert n[4] == 4 and toks[4, 4] == 1500          # smallest j with (j + 1) / 3000 > 0.5
    # block 4's draw lands on a boundary of the uniform CDF: unpinned for the oracle
    assert check(inp, n, toks) <= 1


def test_workspace_reused_and_graph_captured(mx):
    import torch
    w = VerifyWorkload("graph", 9000, 8, 3)
    inps = [verify_inputs(w, seed=s) for s in (21, 22)]
    sv = mx.SpecVerify(3, 8, 9000)
    ref = [_run(mx, inp, sv) for inp in inps]
    for inp, (n, toks) in zip(inps, ref):
        assert check(inp, n, toks) == 0
    ts = [_dev(inp) for inp in inps]
    outs = [(torch.empty(3, dtype=torch.int32, device="cuda"), torch.empty((3, 9), dtype=torch.int32, device="cuda"))
            for _ in ts]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for t, (n, k) in zip(ts, outs):
            sv(t["lt"], t["ld"], t["d"], t["r"], t["u"], n_out=n, tokens_out=k)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    sv.status()
    for (n, k), (rn, rk) in zip(outs, ref):
        assert (n.cpu().numpy() == rn).all() and (k.cpu().numpy() == rk).all()


def test_exp_within_two_ulp(mx):
    """The step's table-driven exp against the host libm (numpy) over the range the
    step uses; 0 below -708 and for -inf."""
    import torch
    rng = np.random.default_rng(1)
    x = np.concatenate([-rng.uniform(0, 708, 200000), -rng.uniform(0, 1, 100000), -rng.exponential(10, 100000),
                        -np.arange(0, 708, 1 / 64.0),
                        [0.0, -0.0, -1e-300, -np.log(2), -707.9, -708.0, -709.0, -1e4, -np.inf]])
    y = mx.spec_exp(torch.from_numpy(x).cuda()).cpu().numpy()
    ref = np.exp(x)
    ok = x > -708
    err = np.abs(y[ok] - ref[ok]) / np.spacing(ref[ok])
    assert err.max() <= 2.0, (err.max(), x[ok][np.argmax(err)])
    assert (y[~ok] == 0).all()
    assert (y[x == 0.0] == 1.0).all()
