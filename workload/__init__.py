"""Seeded synthetic inputs for absorbed MLA latent decode.

This module describes the five decode workloads (their shapes and value
distributions) and draws their inputs.  It holds none of the method's
arithmetic: it only draws random numbers, rounds them to bf16, builds context
lengths and shuffled page tables.  The CPU oracle and the CUDA path are both
fed from here, byte for byte, and nothing else is shared between them.

Value distributions follow the workloads' description: activations (the hidden
state h and the query q) are N(0, 1); weights are N(0, 1/fan_in) with fan_in =
d_model for the joint down-projection [W_DKV; W_KR] and fan_in = d_c for the
per-head up-projections W_UK and W_UV (the in_features of the nn.Linear layers in
the distaisys.com deep-dive, section 3 "PyTorch Reference Implementation");
prefilled latent-cache rows (c_KV and the already-rotated k_R) are N(0, 1).

Every tensor has its own PCG64 stream keyed by (seed, tensor name), so adding a
tensor never shifts another one's values.  bf16 conversion rounds to nearest,
ties to even.
"""
from __future__ import annotations

import dataclasses
import zlib

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "DecodeInputs", "bf16_bits", "bf16_to_f32",
    "rng_for", "context_lengths", "make_page_table", "make_decode_inputs",
    "make_out_proj_inputs", "make_query_proj_inputs", "Q_LORA_RANK",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one decode step of one attention layer."""
    name: str
    batch: int                 # B sequences
    nq: int                    # query tokens per sequence in this step
    n_heads: int               # H
    d_model: int               # D
    d_c: int                   # latent width (kv_lora_rank)
    d_rope: int                # decoupled RoPE key width
    qk_nope: int               # per-head non-rotary query/key width (d_h)
    v_head: int                # per-head value width
    page_size: int = 64        # tokens per latent-cache page
    context: int | None = None     # uniform context length N (after this step's append)
    ragged: tuple[int, int] | None = None  # inclusive range of per-sequence N
    shuffle_pages: bool = True
    rope_theta: float = 10000.0
    fp32_values: bool = False  # the tiny case is specified in fp32

    @property
    def row(self) -> int:
        """Cache row width: latent c_KV followed by the rotated RoPE key."""
        return self.d_c + self.d_rope

    @property
    def tokens(self) -> int:
        return self.batch * self.nq


WORKLOADS: dict[str, Workload] = {
    # Tiny: batch 1, one query token, 4 heads, cache length 128, fp32 values.
    "tiny": Workload("tiny", batch=1, nq=1, n_heads=4, d_model=256, d_c=64, d_rope=16,
                     qk_nope=32, v_head=32, context=128, shuffle_pages=False,
                     fp32_values=True),
    # DeepSeek-V2-shaped: 8 sequences of 4096, 32 heads.
    "v2": Workload("v2", batch=8, nq=1, n_heads=32, d_model=4096, d_c=512, d_rope=64,
                   qk_nope=128, v_head=128, context=4096),
    # DeepSeek-V3-shaped: 16 sequences of 32768, 128 heads.
    "v3": Workload("v3", batch=16, nq=1, n_heads=128, d_model=7168, d_c=512, d_rope=64,
                   qk_nope=128, v_head=128, context=32768),
    # Long context: 8 sequences of 131072, 128 heads.
    "long": Workload("long", batch=8, nq=1, n_heads=128, d_model=7168, d_c=512, d_rope=64,
                     qk_nope=128, v_head=128, context=131072),
    # Ragged serving batch: 64 sequences, N ~ U[1024, 65536], 2 query tokens each.
    "ragged": Workload("ragged", batch=64, nq=2, n_heads=128, d_model=7168, d_c=512,
                       d_rope=64, qk_nope=128, v_head=128, ragged=(1024, 65536)),
}


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def rng_for(seed: int, name: str) -> np.random.Generator:
    """Independent PCG64 stream for one named tensor of one seed."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, zlib.crc32(name.encode())])))


def _normal(seed: int, name: str, shape, std: float = 1.0) -> np.ndarray:
    g = rng_for(seed, name)
    out = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def _normal_bf16(seed: int, name: str, shape, chunk: int = 1 << 22, std: float = 1.0) -> np.ndarray:
    """N(0, std^2) draws rounded to bf16 for the large tensors (latent-cache
    pools, the output projection).

    The tensor is cut into chunks of `chunk` elements; chunk k draws from its own
    PCG64 stream keyed by (seed, name, k), so the values do not depend on how many
    threads fill them (numpy releases the GIL while it draws).
    """
    import concurrent.futures
    import os
    out = np.empty(int(np.prod(shape)), dtype=np.uint16)
    key = zlib.crc32(name.encode())

    def fill(k):
        s = k * chunk
        n = min(chunk, out.size - s)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, key, k])))
        v = g.standard_normal(size=n, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[s:s + n] = bf16_bits(v)

    nchunks = (out.size + chunk - 1) // chunk
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


def context_lengths(w: Workload, seed: int) -> np.ndarray:
    """Per-sequence context length N_b after this step's append (int32 [B])."""
    if w.context is not None:
        return np.full(w.batch, w.context, dtype=np.int32)
    lo, hi = w.ragged
    return rng_for(seed, "context_lengths").integers(lo, hi, size=w.batch, endpoint=True).astype(np.int32)


def make_page_table(lens: np.ndarray, page_size: int, seed: int, shuffle: bool,
                    spare_pages: int = 0, max_pages: int | None = None):
    """Page table for sequences of the given lengths.

    Sequence b owns ceil(N_b / page_size) pages.  Physical page ids are a
    permutation of range(num_pages) (Fisher-Yates shuffle from the seed when
    `shuffle`), handed out in order.  Unused table entries hold -1.  `spare_pages`
    extra physical pages are allocated and never referenced (canaries).
    Returns (page_table int32 [B, max_pages], num_pages).
    """
    need = [(int(n) + page_size - 1) // page_size for n in lens]
    total = sum(need)
    num_pages = total + spare_pages
    ids = np.arange(num_pages, dtype=np.int32)
    if shuffle:
        ids = rng_for(seed, "page_permutation").permutation(ids).astype(np.int32)
    width = max(need) if max_pages is None else max_pages
    table = np.full((len(lens), max(width, 1)), -1, dtype=np.int32)
    k = 0
    for b, n in enumerate(need):
        table[b, :n] = ids[k:k + n]
        k += n
    return table, num_pages


@dataclasses.dataclass
class DecodeInputs:
    """All inputs of one decode step.  Float tensors are kept as bf16 bits
    (`bits[name]`, uint16) and, for the fp32-specified tiny case, also as the
    unrounded float32 draws (`raw[name]`)."""
    workload: Workload
    seed: int
    lens: np.ndarray          # int32 [B]  context length after this step's append
    seq_idx: np.ndarray       # int32 [T]  sequence of each query token
    pos: np.ndarray           # int32 [T]  cache index (= RoPE position) of each query token
    h_seq_idx: np.ndarray     # int32 [Ta] sequence of each appended token
    h_pos: np.ndarray         # int32 [Ta] cache index of each appended token
    page_table: np.ndarray    # int32 [B, max_pages]
    num_pages: int
    bits: dict                # name -> uint16 array (bf16)
    raw: dict                 # name -> float32 array (unrounded), fp32 workloads only

    def f64(self, name: str) -> np.ndarray:
        """bf16 values of a tensor, widened to float64."""
        return bf16_to_f32(self.bits[name]).astype(np.float64)


def make_decode_inputs(w: Workload, seed: int = 0, spare_pages: int = 0,
                       prefill: bool = True, max_pages: int | None = None,
                       append_all: bool = False, lens=None) -> DecodeInputs:
    """Draw every input of one decode step of workload `w`.

    Tensors (bf16 bits):
      h      [T, D]                 hidden states of the tokens appended this step
      q      [T, H, qk_nope+d_rope] projected queries (non-rotary part first)
      w_dkv  [d_c+d_rope, D]        rows 0..d_c-1 = W_DKV, rows d_c.. = W_KR
      w_uk   [H, qk_nope, d_c]      key up-projection per head
      w_uv   [H, v_head, d_c]       value up-projection per head
      pool   [num_pages, page, d_c+d_rope]  paged latent cache; rows of earlier
             tokens prefilled with N(0,1), the rest random (overwritten by append)
    Query token t belongs to sequence t // nq and sits at cache index N_b - nq + t % nq.
    By default the appended tokens are the query tokens (Ta = T).  With
    `append_all` every cache row of every sequence is appended this step
    (Ta = sum N_b, pool starts zeroed): the tiny case builds its whole cache so.
    `lens` overrides the per-sequence context lengths of the workload.
    """
    lens = context_lengths(w, seed) if lens is None else np.asarray(lens, dtype=np.int32)
    assert lens.shape == (w.batch,) and (lens >= w.nq).all()
    T = w.tokens
    seq_idx = np.repeat(np.arange(w.batch, dtype=np.int32), w.nq)
    pos = (lens[seq_idx] - w.nq + np.tile(np.arange(w.nq, dtype=np.int32), w.batch)).astype(np.int32)
    table, num_pages = make_page_table(lens, w.page_size, seed, w.shuffle_pages, spare_pages, max_pages)
    if append_all:
        h_seq_idx = np.concatenate([np.full(n, b, dtype=np.int32) for b, n in enumerate(lens)])
        h_pos = np.concatenate([np.arange(n, dtype=np.int32) for n in lens])
        prefill = False
    else:
        h_seq_idx, h_pos = seq_idx.copy(), pos.copy()

    raw = {
        "h": _normal(seed, "h", (len(h_pos), w.d_model)),
        "q": _normal(seed, "q", (T, w.n_heads, w.qk_nope + w.d_rope)),
        "w_dkv": _normal(seed, "w_dkv", (w.row, w.d_model), std=1.0 / np.sqrt(w.d_model)),
        "w_uk": _normal(seed, "w_uk", (w.n_heads, w.qk_nope, w.d_c), std=1.0 / np.sqrt(w.d_c)),
        "w_uv": _normal(seed, "w_uv", (w.n_heads, w.v_head, w.d_c), std=1.0 / np.sqrt(w.d_c)),
    }
    bits = {k: bf16_bits(v) for k, v in raw.items()}
    pool_shape = (num_pages, w.page_size, w.row)
    if prefill and w.fp32_values:
        raw["pool"] = _normal(seed, "pool", pool_shape)
        bits["pool"] = bf16_bits(raw["pool"])
    elif prefill:
        bits["pool"] = _normal_bf16(seed, "pool", pool_shape)
    else:
        bits["pool"] = np.zeros(pool_shape, dtype=np.uint16)
    if not w.fp32_values:
        raw = {}
    return DecodeInputs(w, seed, lens, seq_idx, pos, h_seq_idx, h_pos, table, num_pages, bits, raw)


# q_lora_rank of the V3-shaped decoder (eyestech.in MLA article, sec. 3)
Q_LORA_RANK = 1536


def make_query_proj_inputs(w: Workload, seed: int = 0, n_tokens: int | None = None,
                           q_lora_rank: int = Q_LORA_RANK) -> dict:
    """Inputs of the q-LoRA query path c_Q = W_DQ h, q = W_UQ c_Q (bf16 bits):
      h     [T, D]                          hidden states, N(0, 1)
      w_dq  [q_lora_rank, D]                N(0, 1/D)
      w_uq  [H * (qk_nope + d_rope), q_lora_rank]   N(0, 1/q_lora_rank)
    (fan_in = in_features, as for the other projections).  T defaults to batch * nq."""
    T = w.tokens if n_tokens is None else int(n_tokens)
    n_q = w.n_heads * (w.qk_nope + w.d_rope)
    return {
        "h": bf16_bits(_normal(seed, "q_path_h", (T, w.d_model))),
        "w_dq": _normal_bf16(seed, "w_dq", (q_lora_rank, w.d_model), std=1.0 / np.sqrt(w.d_model)),
        "w_uq": _normal_bf16(seed, "w_uq", (n_q, q_lora_rank), std=1.0 / np.sqrt(q_lora_rank)),
    }


def make_out_proj_inputs(w: Workload, seed: int = 0, n_tokens: int | None = None) -> dict:
    """Inputs of the layer output projection y = W_O concat_h(o_h) (bf16 bits):
      o    [T, H, v_head]       the heads' attention outputs, N(0, 1)
      w_o  [D, H * v_head]      out_proj weight, N(0, 1/fan_in) with fan_in = H * v_head
                                (in_features of out_proj, distaisys.com deep-dive sec. 3)
    T defaults to the workload's query tokens (batch * nq)."""
    T = w.tokens if n_tokens is None else int(n_tokens)
    K = w.n_heads * w.v_head
    return {
        "o": bf16_bits(_normal(seed, "attn_out", (T, w.n_heads, w.v_head))),
        "w_o": _normal_bf16(seed, "w_o", (w.d_model, K), std=1.0 / np.sqrt(K)),
    }
