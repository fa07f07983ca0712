"""CPU oracle for the Hy-Nomas segment-causal attention over an INT8 KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, link or run
anything in this package: only the tests, the package's smoke check and the
benchmark's CPU-baseline / reference arm call it.  It shares no code with the
CUDA path (no kernels, headers, tables or helpers); the only thing both sides
consume is the seeded input generator in `int8_kv_cache_action_b200.workloads`,
which holds no arithmetic of the method.

What it computes, and the passages it follows (pages cited by site and section):

* `quant`      -- INT8 storage with a float scale per (token, head) and BF16
                  compute: fluxbbs.com "单卡 4090 怎么做到的" (first technique:
                  weights and cached keys/values stored as INT8 with float scale
                  factors, dequantised to BF16 for compute).  fp32, bit-exact.
* `ring`       -- the 18-latent-frame sliding history window (same section,
                  second technique; hyphentech.top config table: "at most 18
                  history latent frames" on the GPU) and the KV cache that each
                  finished segment is written into for the next segment
                  (fluxbbs.com "架构").
* `visibility` -- segment-causal attention plus the action-aware mask:
                  description heads visible across segments, action tails
                  visible only in their own segment and their time window
                  (fluxbbs.com "架构", second paragraph pair).
* `select`     -- block-sparse mode: after the first two denoising steps only
                  25 % of candidate video blocks are kept (fluxbbs.com
                  "单卡 4090 怎么做到的", fourth technique).  The ranking rule
                  (mean-pooled q . mean-pooled k in a fixed fp32 order) is this
                  project's own definition; the pages fix only the fraction.
* `attention`  -- softmax attention over the visible keys in fp64.

Parity status: every function here is pinned by the `-m "not gpu"` tests in
tests/test_oracle_*.py (closed forms, invariants, reductions to library
routines, brute force on tiny inputs).  The real system's sparse ranking rule
is unknown, so "parity vs the real system" for `select` is unpinned; the
oracle's own definition is what the CUDA path must match bit for bit.
"""
from . import quant, ring, visibility, select, attention  # noqa: F401

__all__ = ["quant", "ring", "visibility", "select", "attention"]
