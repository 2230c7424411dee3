"""CPU oracle for the MXFP4 MoE expert feed-forward: TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 restatement of what the decode-time MoE path computes, used
to check the CUDA path.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the
product path (the C-ABI library and its Python binding) never does, and shares
no code with it.

Sources.  The pages on MiMo-V2.5-Pro-UltraSpeed / TileRT name the format and
the policy only: expert weights in MXFP4 at 4 bits per parameter, everything
else, routing included, kept at higher precision (bjdmk.com.cn news, section
"极致协同，通向千速之路"; yifor blog digest "Xiaomi MiMo and TileRT Push a
1-Trillion-Parameter Model Past 1000 Tokens Per Second on Commodity GPUs",
section "三層協同設計"; sandbot blog "1000 TPS paradigm", section
"三、技术拆解：怎么做到的？").  The block layout (32 E2M1 codes sharing one
E8M0 scale, scale = floor(log2 amax) - 2) is the OCP Microscaling (MX) v1.0
specification's MXFP4; softmax/top-k/renormalise routing and SwiGLU experts
are the plainest reading of an MoE decoder layer where the pages are silent.

Modules:
  mxfp4  E2M1/E8M0 decode, dequantise, the reference quantiser;
  moe    router, permutation, expert FFN, weighted combine, RMSNorm, chain.

Every function here has at least one pin in ``tests/test_oracle_*.py`` that
does not go through the function itself (tables, closed forms, brute force,
invariants); no function is "parity unpinned".
"""
from . import mxfp4, moe  # noqa: F401
