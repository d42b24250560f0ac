"""CPU oracle for absorbed MLA latent decode.

TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the
benchmark's CPU-baseline / reference leg are the only callers allowed.  The
product path (the CUDA library and its Python binding) never imports, calls or
links anything in this package, and this package imports nothing from the
product path.

Contents:
  mla.py               the decode step in float64: KV-row append (W_DKV, W_KR,
                       RoPE), the naive decompressing attention (the parity
                       authority), the absorbed form, a brute-force loop form,
                       split-KV partials with a log-sum-exp merge, and paged
                       cache gathering.
  cache_accounting.py  closed-form KV-cache sizes per architecture.

Every function says which page and section it follows.  Pages cited:
  [eyestech-pypi]  "eyestech-mla 1.0.0" package description (PyPI)
  [eyestech-blog]  "DeepSeek MLA Architecture: How It Cuts KV Cache by 93%" (eyestech.in)
  [from-scratch]   "mla-from-scratch" README (github, aghasalim)
  [distaisys]      "Deep-Dive: Multi-Head Latent Attention (MLA) and Low-Rank KV Cache
                   Compression in DeepSeek-V3" (distaisys.com)
  [songhuiming]    "MHA vs MLA KV cache comparison" (songhuiming.github.io, 2025-08-01)

Parity status: every function here is pinned by a `-m "not gpu"` test against
closed forms, hand-derived fixtures, invariants or brute force (tests/test_oracle_*.py).
"""
from . import mla, cache_accounting  # noqa: F401
