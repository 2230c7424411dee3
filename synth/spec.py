"""Seeded synthetic inputs for the speculative-verify acceptance step.

This module only draws random numbers. It holds none of the acceptance
step's arithmetic: no softmax, no acceptance test, no residual distribution
and no sampling. Both the CPU oracle and the CUDA path consume what it
produces.

Recipe, per verify block b (one sequence) and position i:

* target logits ``lt[b][i]`` (i = 0 .. G, fp32, V entries): sigma * N(0, 1),
  plus a boost drawn from U[peak_lo, peak_hi] added to one leading token,
  itself drawn uniformly from the vocabulary. The softmax of such a row puts
  between about 10% and 95% of its mass on the leading token, and spreads
  the rest over a long tail;
* draft logits ``ld[b][i]`` (i = 0 .. G-1, fp32): the target row of the same
  position plus draft_noise * N(0, 1), so the draft distribution is close to
  the target's but not equal to it;
* draft tokens ``d[b][i]``: the draft model's own samples from its logits,
  drawn by the Gumbel-max rule (the index of the largest ld + Gumbel(0, 1)
  noise);
* uniforms ``r[b][i]`` (acceptance tests) and ``u[b]`` (the one sample the
  step draws), fp64 in [0, 1). They are the random numbers of the method,
  passed in as inputs.

Each tensor has its own numpy PCG64 stream. The stream's seed comes from
the SHA-256 of (seed, block range, kind).
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass

import numpy as np

__all__ = ["VerifyWorkload", "VERIFY_WORKLOADS", "verify_inputs"]


@dataclass(frozen=True)
class VerifyWorkload:
    """Verify blocks of gamma draft tokens over a vocabulary of `vocab` entries."""
    name: str
    vocab: int
    gamma: int
    blocks: int
    logit_sigma: float = 2.0
    peak_lo: float = 13.0
    peak_hi: float = 18.0
    draft_noise: float = 0.25

    def with_blocks(self, b: int) -> "VerifyWorkload":
        return VerifyWorkload(self.name, self.vocab, self.gamma, b, self.logit_sigma, self.peak_lo,
                              self.peak_hi, self.draft_noise)


# The pages' block size is 8 draft tokens. They give no vocabulary size;
# 152,064 entries is taken, of the order of large-LLM vocabularies. A single
# sequence is the latency case. 64 sequences give the throughput case.
VERIFY_WORKLOADS = {
    "verify_tiny_v1000_g8": VerifyWorkload("verify_tiny_v1000_g8", 1000, 8, 4),
    "verify_b1_v152064_g8": VerifyWorkload("verify_b1_v152064_g8", 152064, 8, 1),
    "verify_b64_v152064_g8": VerifyWorkload("verify_b64_v152064_g8", 152064, 8, 64),
}


def _rng(seed: int, kind: str, b0: int, b1: int) -> np.random.Generator:
    tag = f"mxfp4-moe/verify/{seed}/{b0}-{b1}/{kind}".encode()
    return np.random.Generator(np.random.PCG64(int.from_bytes(hashlib.sha256(tag).digest()[:8], "little")))


def verify_inputs(w: VerifyWorkload, seed: int = 0) -> dict:
    """Inputs of w.blocks verify blocks: lt [B][G+1][V] f32, ld [B][G][V] f32,
    d [B][G] i32, r [B][G] f64, u [B] f64."""
    B, G, V = w.blocks, w.gamma, w.vocab
    lt = (_rng(seed, "target", 0, B).standard_normal((B, G + 1, V), dtype=np.float32)
          * np.float32(w.logit_sigma))
    pk = _rng(seed, "peak", 0, B)
    lead = pk.integers(0, V, size=(B, G + 1))
    boost = pk.uniform(w.peak_lo, w.peak_hi, size=(B, G + 1)).astype(np.float32)
    bi, ii = np.meshgrid(np.arange(B), np.arange(G + 1), indexing="ij")
    lt[bi, ii, lead] += boost
    ld = lt[:, :G] + (_rng(seed, "draft", 0, B).standard_normal((B, G, V), dtype=np.float32)
                      * np.float32(w.draft_noise))
    gum = _rng(seed, "gumbel", 0, B)
    d = np.empty((B, G), dtype=np.int32)
    for b in range(B):
        g = -np.log(-np.log(gum.uniform(np.finfo(np.float64).tiny, 1.0, size=(G, V))))
        d[b] = np.argmax(ld[b].astype(np.float64) + g, axis=1)
    r = _rng(seed, "r", 0, B).uniform(0.0, 1.0, size=(B, G))
    u = _rng(seed, "u", 0, B).uniform(0.0, 1.0, size=(B,))
    return {"lt": np.ascontiguousarray(lt), "ld": np.ascontiguousarray(ld), "d": d, "r": r, "u": u}
