"""Closed-form KV-cache sizes (TEST INFRASTRUCTURE ONLY; see the package docstring).

Elements stored per token per layer:
  MHA with n_h heads of width d_h:   2 * n_h * d_h (a key and a value per head)
  GQA with group size g:             2 * (n_h / g) * d_h
  MQA:                               2 * d_h
  MLA with decoupled RoPE:           d_c + d_rope (one latent and one shared RoPE key)
  MLA without decoupled RoPE:        d_c
([from-scratch] "The problem" table; [eyestech-pypi] "Key Architectural
Highlights" table; [songhuiming] "Cache Size (MLA)" and "Side-by-side Comparison".)

Bytes = elements/token/layer * tokens * layers * batch * bytes per element.  The
pages print sizes in binary units: their "GB" is 2^30 bytes and [songhuiming]'s
"MB" is 2^20 bytes.
"""
from __future__ import annotations

GIB = 1 << 30
MIB = 1 << 20


def elements_per_token_layer(arch: str, *, n_heads: int = 0, d_head: int = 0,
                             group: int = 1, d_c: int = 0, d_rope: int = 0) -> int:
    """Scalars cached per token per layer for one attention architecture."""
    if arch == "mha":
        return 2 * n_heads * d_head
    if arch == "gqa":
        assert n_heads % group == 0
        return 2 * (n_heads // group) * d_head
    if arch == "mqa":
        return 2 * d_head
    if arch == "mla":
        return d_c + d_rope
    if arch == "mla_no_rope":
        return d_c
    raise ValueError(arch)


def compute_kv_cache_bytes(n_layers: int, n_kv_heads: int, d_head: int, seq_len: int,
                           batch_size: int, bytes_per_elem: int, is_mla: bool = False,
                           d_latent: int = 512, d_rope: int = 64) -> int:
    """KV-cache bytes of a whole model, with the argument list of the
    `compute_kv_cache_bytes` call shown in [eyestech-pypi] "Programmatic Memory
    Benchmark API": MLA stores d_latent + d_rope scalars per token per layer,
    MHA/GQA store 2 * n_kv_heads * d_head."""
    if is_mla:
        per_tok = elements_per_token_layer("mla", d_c=d_latent, d_rope=d_rope)
    else:
        per_tok = 2 * n_kv_heads * d_head
    return per_tok * seq_len * n_layers * batch_size * bytes_per_elem


def format_gb(nbytes: int) -> str:
    """Bytes in the pages' "GB" (2^30 bytes), two decimals."""
    return f"{nbytes / GIB:.2f} GB"


def compression_vs(elements_a: int, elements_b: int) -> float:
    """How many times fewer scalars b stores than a (the "vs MHA" column)."""
    return elements_a / elements_b


def reduction_fraction(elements_base: int, elements_new: int) -> float:
    """Fraction of the cache removed: 1 - new/base."""
    return 1.0 - elements_new / elements_base
