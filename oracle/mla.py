"""Float64 CPU oracle of one MLA decode step over a paged latent cache.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Plain numpy, float64
throughout, no blocking or fusion beyond what each definition states.

Notation (pages' symbols):
  h_t      hidden state of token t, length D
  c_t      latent KV vector, c_t = W_DKV h_t, length d_c          [distaisys] sec. 2
  k_t^R    decoupled RoPE key, one per token shared by all heads,
           k_t^R = RoPE(W_KR h_t, t), length d_rope               [eyestech-pypi] "Key
           Architectural Highlights" item 2; [from-scratch] "Absorption, and why RoPE breaks it"
  cache row  [c_t || k_t^R], 576 = 512 + 64 scalars                [eyestech-pypi] item 2
  K_{n,h}  = W_UK,h c_n  (d_h),  V_{n,h} = W_UV,h c_n  (d_v)        [distaisys] sec. 2
  q~_h     = W_UK,h^T q_nope,h  (absorbed query, length d_c)       [eyestech-blog] sec. 2;
                                                                    [eyestech-pypi] item 3
Weight layouts (nn.Linear weight convention, [out, in], [distaisys] sec. 3):
  w_dkv [d_c + d_rope, D]   rows 0..d_c-1 are W_DKV, the last d_rope rows W_KR
  w_uk  [H, d_h, d_c]       w_uk[h] = W_UK,h
  w_uv  [H, d_v, d_c]       w_uv[h] = W_UV,h
Query q [T, H, d_h + d_rope]: per head the non-rotary part q_nope first, then
the rotary part q_rope (not yet rotated).

Readings where the pages are silent (each is listed in the design notes):
  * RoPE pairs adjacent channels (2i, 2i+1) and rotates them by
    pos * theta^(-2i/d_rope), theta = 10000 (RoFormer, which [from-scratch] cites
    for RoPE and its relative-position property).
  * A token's RoPE position is its cache index; a query sits at the index where
    its own latent row is appended, and attends to every key index <= its own
    (the cache is appended before attending: [songhuiming] "MLA ... Step-by-step",
    [eyestech-pypi] quickstart, cache 1024 -> 1025).
  * Softmax scale 1/sqrt(d_h + d_rope): the query/key width once the RoPE part is
    concatenated ([distaisys] sec. 3 scales by 1/sqrt(d_h) without RoPE).
  * lse is the natural-log log-sum-exp of the scaled scores.
"""
from __future__ import annotations

import math

import numpy as np

DEFAULT_THETA = 10000.0


def softmax_scale(d_h: int, d_rope: int) -> float:
    """1/sqrt(d_h + d_rope): scaled dot-product attention ([distaisys] sec. 3,
    [songhuiming] "softmax(q K^T / sqrt(d_h))") over the concatenated
    non-rotary + rotary query/key of width d_h + d_rope."""
    return 1.0 / math.sqrt(d_h + d_rope)


def rope(x: np.ndarray, pos, theta: float = DEFAULT_THETA) -> np.ndarray:
    """Rotary position embedding on the last axis of `x` (even width d).

    Channel pair (2i, 2i+1), i = 0 .. d/2-1, is rotated by the angle
    pos * theta^(-2i/d):  (a, b) -> (a cos - b sin, a sin + b cos).
    `pos` broadcasts against x.shape[:-1].
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    assert d % 2 == 0
    i = np.arange(d // 2, dtype=np.float64)
    freq = theta ** (-2.0 * i / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq
    cos, sin = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)), dtype=np.float64)
    out[..., 0::2] = a * cos - b * sin
    out[..., 1::2] = a * sin + b * cos
    return out


# ----------------------------------------------------------------------------
# Cache append: c_t = W_DKV h_t, k_t^R = RoPE(W_KR h_t, t)
# ----------------------------------------------------------------------------

def kv_rows(h: np.ndarray, w_dkv: np.ndarray, pos: np.ndarray, d_c: int,
            theta: float = DEFAULT_THETA) -> np.ndarray:
    """Cache rows [c_t || k_t^R] for tokens h [T, D] at positions pos [T].

    c_t = W_DKV h_t ([distaisys] sec. 2; [songhuiming] "Down-project to
    compressed latent"), k^_t = W_KR h_t, k_t^R = RoPE(k^_t, t).  Returns [T, d_c + d_rope].
    """
    h = np.asarray(h, dtype=np.float64)
    w = np.asarray(w_dkv, dtype=np.float64)
    c = h @ w[:d_c].T
    k_hat = h @ w[d_c:].T
    k_r = rope(k_hat, np.asarray(pos), theta)
    return np.concatenate([c, k_r], axis=-1)


def page_slot(page_table: np.ndarray, b: int, n: int, page_size: int) -> tuple[int, int]:
    """Physical (page, slot) of cache index n of sequence b."""
    return int(page_table[b, n // page_size]), n % page_size


def append_rows(pool: np.ndarray, page_table: np.ndarray, seq_idx, pos, rows) -> None:
    """Write cache rows into the paged pool [num_pages, page, row] in place."""
    page_size = pool.shape[1]
    for t in range(len(pos)):
        p, s = page_slot(page_table, int(seq_idx[t]), int(pos[t]), page_size)
        pool[p, s, :] = rows[t]


def gather_cache(pool: np.ndarray, table_row: np.ndarray, n: int) -> np.ndarray:
    """Logical cache rows 0..n-1 of one sequence, read through its page-table row."""
    page_size = pool.shape[1]
    idx = np.arange(n)
    return pool[table_row[idx // page_size], idx % page_size]


# ----------------------------------------------------------------------------
# Query absorption: q~_h = W_UK,h^T q_nope,h ; q_r = RoPE(q_rope,h, pos)
# ----------------------------------------------------------------------------

def absorb_queries(q: np.ndarray, pos: np.ndarray, w_uk: np.ndarray,
                   theta: float = DEFAULT_THETA) -> np.ndarray:
    """Absorbed queries q_lat [T, H, d_c + d_rope] = [W_UK,h^T q_nope || RoPE(q_rope, pos)].

    The content score q . k_n = q . (W_UK c_n) = (W_UK^T q) . c_n by associativity
    ([from-scratch] "Absorption, and why RoPE breaks it"; [eyestech-blog] sec. 2).
    """
    q = np.asarray(q, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    d_h = w_uk.shape[1]
    q_nope, q_rope = q[..., :d_h], q[..., d_h:]
    # q~[t, h, j] = sum_i W_UK,h[i, j] q_nope[t, h, i]
    q_tilde = np.einsum("hij,thi->thj", w_uk, q_nope)
    q_r = rope(q_rope, np.asarray(pos)[:, None], theta)
    return np.concatenate([q_tilde, q_r], axis=-1)


# ----------------------------------------------------------------------------
# Attention of one query token over n cached tokens
# ----------------------------------------------------------------------------

def attend_naive(q: np.ndarray, q_pos: int, C: np.ndarray, KR: np.ndarray,
                 w_uk: np.ndarray, w_uv: np.ndarray, scale: float,
                 theta: float = DEFAULT_THETA):
    """Naive (decompressing) MLA attention of one query token, all heads.

    Per head h: K_n = W_UK,h c_n and V_n = W_UV,h c_n are materialised for every
    cached token ([distaisys] sec. 2-3; [songhuiming] "Up-project ALL cached
    latents to K, V"), the full key is [K_n || k_n^R] and the full query
    [q_nope || RoPE(q_rope, q_pos)]; s_n = scale * q_full . k_full_n, p =
    softmax(s), o_h = sum_n p_n V_n.

    q [H, d_h + d_rope]; C [n, d_c]; KR [n, d_rope] (already rotated).
    Returns o [H, d_v] and lse [H] (natural log).
    """
    q = np.asarray(q, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    KR = np.asarray(KR, dtype=np.float64)
    H, d_h = w_uk.shape[0], w_uk.shape[1]
    d_v = w_uv.shape[1]
    o = np.empty((H, d_v))
    lse = np.empty(H)
    for h in range(H):
        K = C @ np.asarray(w_uk[h], dtype=np.float64).T        # [n, d_h]
        V = C @ np.asarray(w_uv[h], dtype=np.float64).T        # [n, d_v]
        k_full = np.concatenate([K, KR], axis=1)
        q_full = np.concatenate([q[h, :d_h], rope(q[h, d_h:], q_pos, theta)])
        s = scale * (k_full @ q_full)
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        o[h] = (e / l) @ V
        lse[h] = m + math.log(l)
    return o, lse


def attend_absorbed(q_lat: np.ndarray, C: np.ndarray, KR: np.ndarray,
                    w_uv: np.ndarray, scale: float):
    """Absorbed MLA attention of one query token, all heads.

    s_n = scale * (q~ . c_n + q_r . k_n^R) (content term + positional term,
    [from-scratch] "Absorption, and why RoPE breaks it"), p = softmax(s), the
    values are read in latent space, o_lat = sum_n p_n c_n, and up-projected once,
    o_h = W_UV,h o_lat ([from-scratch], same section, value side).

    q_lat [H, d_c + d_rope]; C [n, d_c]; KR [n, d_rope].  Returns o [H, d_v], lse [H].
    """
    o_lat, lse = attend_latent(q_lat, C, KR, scale)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    o = np.einsum("hvc,hc->hv", w_uv, o_lat)
    return o, lse


def attend_latent(q_lat: np.ndarray, C: np.ndarray, KR: np.ndarray, scale: float):
    """Latent-space part of the absorbed form: o_lat [H, d_c] (softmax-weighted
    mean of the cached latents) and lse [H].  An empty cache gives o_lat = 0 and
    lse = -inf (a split that sees no key contributes nothing)."""
    q_lat = np.asarray(q_lat, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    KR = np.asarray(KR, dtype=np.float64)
    d_c = C.shape[1]
    H = q_lat.shape[0]
    if C.shape[0] == 0:
        return np.zeros((H, d_c)), np.full(H, -np.inf)
    s = scale * (C @ q_lat[:, :d_c].T + KR @ q_lat[:, d_c:].T)   # [n, H]
    m = s.max(axis=0)
    e = np.exp(s - m)
    l = e.sum(axis=0)
    o_lat = (e / l).T @ C                                        # [H, d_c]
    return o_lat, m + np.log(l)


def attend_brute(q, q_pos, C, KR, w_uk, w_uv, scale, theta=DEFAULT_THETA):
    """Brute-force attention with plain Python loops, for tiny shapes only.

    No max subtraction and no matrix routine: every key and value element is
    an explicit sum, and p_n = exp(s_n) / sum_m exp(s_m) directly.
    Returns o [H][d_v] and lse [H] as nested lists of floats.
    """
    H, d_h, d_c = len(w_uk), len(w_uk[0]), len(w_uk[0][0])
    d_v = len(w_uv[0])
    n = len(C)
    d_r = len(KR[0]) if n else 0
    out, lses = [], []
    for h in range(H):
        q_rot = [float(v) for v in rope(np.array(q[h][d_h:], dtype=np.float64), q_pos, theta)]
        scores = []
        for t in range(n):
            acc = 0.0
            for i in range(d_h):
                k_i = 0.0
                for j in range(d_c):
                    k_i += float(w_uk[h][i][j]) * float(C[t][j])
                acc += float(q[h][i]) * k_i
            for r in range(d_r):
                acc += q_rot[r] * float(KR[t][r])
            scores.append(scale * acc)
        z = sum(math.exp(s) for s in scores)
        row = []
        for v in range(d_v):
            acc = 0.0
            for t in range(n):
                val = 0.0
                for j in range(d_c):
                    val += float(w_uv[h][v][j]) * float(C[t][j])
                acc += math.exp(scores[t]) / z * val
            row.append(acc)
        out.append(row)
        lses.append(math.log(z))
    return out, lses


# ----------------------------------------------------------------------------
# Query path with low-rank query compression (q-LoRA)
# ----------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (8 significant bits,
    ties to even), returned as float64.  One rounding straight from float64.
    Normal range only (|x| >= 2^-126 or 0); inf and nan pass through."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                              # x = m 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)    # np.rint: half to even
    return np.where(np.isfinite(x), r, x)


def query_project(h: np.ndarray, w_dq: np.ndarray, w_uq: np.ndarray, n_heads: int,
                  latent_bf16: bool = True):
    """Queries from the hidden state through the compressed query latent.

    c_Q = W_DQ h (width q_lora_rank, 1536 in the V3-shaped configuration of
    [eyestech-blog] sec. 3), then [q_nope || q_rope] = W_UQ c_Q for every head
    ([songhuiming] "Note on Actual Implementation": the query side is also
    down-projected, then up-projected).  The pages name no normalisation
    between the two maps; none is applied.  With latent_bf16, c_Q is rounded to
    bf16 before the up-projection, as in the bf16 module of [eyestech-blog] sec. 3.

    h [T, D]; w_dq [d_cq, D]; w_uq [H * (d_h + d_rope), d_cq] (rows head-major,
    per head the non-rotary rows first).  Returns (c_q [T, d_cq],
    q [T, H, d_h + d_rope]); q's RoPE part is not rotated yet.
    """
    h = np.asarray(h, dtype=np.float64)
    c_q = h @ np.asarray(w_dq, dtype=np.float64).T
    if latent_bf16:
        c_q = round_bf16(c_q)
    q = c_q @ np.asarray(w_uq, dtype=np.float64).T
    return c_q, q.reshape(h.shape[0], n_heads, q.shape[1] // n_heads)


# ----------------------------------------------------------------------------
# Layer output projection
# ----------------------------------------------------------------------------

def out_project(o: np.ndarray, w_o: np.ndarray) -> np.ndarray:
    """Layer output y[t] = W_O concat_h(o[t, h]).

    [distaisys] sec. 3: the attention output of every head is laid side by side,
    head after head (input index h * d_v + j), and one bias-free linear map of
    width H * d_v -> d_model produces the layer output.  [from-scratch]
    "Absorption, and why RoPE breaks it": on the value side W_UV is applied once
    after attending over the latents, right before this map, so the two fold into
    one matrix by associativity.

    o [T, H, d_v]; w_o [d_model, H * d_v] ([out, in]).  Returns y [T, d_model].
    """
    o = np.asarray(o, dtype=np.float64)
    x = o.reshape(o.shape[0], o.shape[1] * o.shape[2])   # head-major concatenation
    return x @ np.asarray(w_o, dtype=np.float64).T


# ----------------------------------------------------------------------------
# Split-KV partials and their log-sum-exp merge
# ----------------------------------------------------------------------------

def split_partials(q_lat, C, KR, scale, bounds):
    """Latent attention over each key range [bounds[i], bounds[i+1]): returns a
    list of (o_lat_s [H, d_c], lse_s [H]) with o_lat_s normalised within its range."""
    return [attend_latent(q_lat, C[a:b], KR[a:b], scale) for a, b in zip(bounds[:-1], bounds[1:])]


def merge_partials(partials):
    """Log-sum-exp merge of split partials: LSE = log sum_s exp(lse_s),
    o_lat = sum_s exp(lse_s - LSE) o_lat_s.  Ranges with lse_s = -inf weigh 0."""
    lses = np.stack([p[1] for p in partials])           # [S, H]
    olat = np.stack([p[0] for p in partials])           # [S, H, d_c]
    m = lses.max(axis=0)
    w = np.exp(lses - m)                                # exp(-inf) = 0
    tot = w.sum(axis=0)
    lse = m + np.log(tot)
    return np.einsum("sh,shc->hc", w / tot, olat), lse


# ----------------------------------------------------------------------------
# One decode step of one layer, end to end
# ----------------------------------------------------------------------------

def decode_step(*, h, h_seq_idx, h_pos, q, q_pos, pool, page_table, lens, nq,
                w_dkv, w_uk, w_uv, d_c, scale=None, theta=DEFAULT_THETA,
                form="naive", heads=None, queries=None):
    """One decode step: append this step's cache rows, then attend.

    1. rows = [W_DKV h_t || RoPE(W_KR h_t, pos_t)] become cache index pos_t of
       sequence seq_idx_t ([songhuiming] "Update latent cache ... then up-project
       ALL cached latents"; [eyestech-pypi] quickstart: the cache grows by one).
    2. For query token i of sequence b (cache index N_b - nq + i) and every head,
       attention over cache indices 0 .. N_b - nq + i (its own row included;
       the later query of the same step is masked: causal within the step).
       Earlier rows are read from the paged pool through the page table.
       form="naive" decompresses K and V per head; form="absorbed" scores on
       latents with q~ = W_UK^T q_nope and up-projects o_lat once by W_UV.
    `pool` is anything indexable as pool[page_ids, slots] -> rows (only the rows
    a query reads are widened to float64).  `heads` (head indices) and `queries`
    (query-token indices) restrict the attention to a sample; other entries of
    the outputs are NaN.

    Returns dict(out [T, H, d_v], lse [T, H], rows [Ta, d_c + d_rope] (the
    appended rows, float64), q_lat [T, H, d_c + d_rope] (absorbed form, else None)).
    """
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    H, d_h = w_uk.shape[0], w_uk.shape[1]
    d_v = w_uv.shape[1]
    d_r = q.shape[-1] - d_h
    if scale is None:
        scale = softmax_scale(d_h, d_r)
    rows = kv_rows(h, w_dkv, np.asarray(h_pos), d_c, theta)
    appended = {}                                   # sequence -> {cache index: row}
    for t in range(len(h_pos)):
        appended.setdefault(int(h_seq_idx[t]), {})[int(h_pos[t])] = rows[t]

    T = q.shape[0]
    heads = list(range(H)) if heads is None else list(heads)
    queries = list(range(T)) if queries is None else list(queries)
    out = np.full((T, H, d_v), np.nan)
    lse = np.full((T, H), np.nan)
    q_lat = absorb_queries(q, np.asarray(q_pos), w_uk, theta) if form == "absorbed" else None
    for t in queries:
        b = t // nq
        p = int(q_pos[t])
        n = p + 1                                   # keys 0 .. p are visible
        assert n <= int(lens[b])
        cache = np.asarray(gather_cache(pool, page_table[b], n), dtype=np.float64)
        for idx, row in appended.get(b, {}).items():
            if idx < n:
                cache[idx] = row
        C, KR = cache[:, :d_c], cache[:, d_c:]
        if form == "naive":
            o, l = attend_naive(q[t, heads], p, C, KR, w_uk[heads], w_uv[heads], scale, theta)
        elif form == "absorbed":
            o, l = attend_absorbed(q_lat[t, heads], C, KR, w_uv[heads], scale)
        else:
            raise ValueError(form)
        out[t, heads] = o
        lse[t, heads] = l
    return {"out": out, "lse": lse, "rows": rows, "q_lat": q_lat}


def attend_paged_latents(*, q_lat, pool, page_table, lens, nq, w_uv, scale,
                         heads=None, queries=None):
    """Absorbed attention given ready absorbed queries q_lat [T, H, d_c + d_rope]
    over the paged pool as it stands (no append).  Query token t of sequence
    b = t // nq sits at cache index N_b - nq + t % nq and sees indices up to it.
    Returns out [T, H, d_v] and lse [T, H] (NaN outside the sample)."""
    q_lat = np.asarray(q_lat, dtype=np.float64)
    T, H = q_lat.shape[0], q_lat.shape[1]
    d_c = np.asarray(w_uv).shape[2]
    d_v = np.asarray(w_uv).shape[1]
    heads = list(range(H)) if heads is None else list(heads)
    queries = list(range(T)) if queries is None else list(queries)
    out = np.full((T, H, d_v), np.nan)
    lse = np.full((T, H), np.nan)
    for t in queries:
        b = t // nq
        n = int(lens[b]) - nq + t % nq + 1
        cache = gather_cache(pool, page_table[b], n).astype(np.float64)
        o, l = attend_absorbed(q_lat[t, heads], cache[:, :d_c], cache[:, d_c:],
                               np.asarray(w_uv)[heads], scale)
        out[t, heads] = o
        lse[t, heads] = l
    return out, lse
