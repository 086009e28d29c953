"""fp64 oracle of the steps either side of decode attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the cpu_baseline / reference leg of ``bench.py`` may import this module; the
CUDA library never calls it and shares no code with it.

What the pages give, and the readings taken where they are silent:

* MLA explainer (mlqm.cn/news/371735) section 2.2: the position branch
  projects its own q^R and k^R and applies RoPE to them; the semantic branch
  (q^C, k^C, v^C from the latents) takes no RoPE; q = [q^C ; q^R] and
  k = [k^C ; k^R].  The pages print no RoPE formula.  Reading: the rotary
  embedding in its original form, consecutive pairs (x[2i], x[2i+1]) turned
  by the angle pos * base^(-2i/d) for a d-wide vector at position pos.  The
  base is a parameter (10000 in the tests).
* MLA explainer section 2.4: only the semantic latent is cached and k^R is
  regenerated from the position.  The cache layout of the decode kernels holds
  [latent ; k^R] per token, the 576-wide row that the MLRA page's absorbed MLA
  form and the benchmark shapes use.  Reading: the cached k^R is the rotated
  one, so appending a token rotates its k^R at the token's position on the way
  into the cache.
* MLRA page (aitntnews.com newId=23265), MLA paragraph: the key
  up-projection W_UK is absorbed into the query at decode time.  With
  k^C_h = W_UK[h] c (W_UK[h] of shape d_h x d_c), q^C_h . k^C_h =
  (q^C_h W_UK[h]) . c, so the absorbed query is q_nope[h] = q^C[h] @ W_UK[h].
* MLA explainer section 2.3: the output weights the semantic values v^C,
  v^C_h = c W_UV[h] (W_UV[h] of shape d_c x d_v), so the head output is the
  attention-weighted latent times W_UV[h].
* MLRA page, block decomposition and "moving the sum outside": the latent
  and its weight matrices are cut into R blocks; each branch is projected and
  attended on its own and the branch outputs are summed.  The up-projection
  of head h therefore takes the R branch outputs side by side against the R
  row blocks of W_UV[h] (one matrix of (R d_c) x d_v), so the branch sum is
  the last part of the contraction.
"""

from __future__ import annotations

import numpy as np

PAGE = 64


def rope_angles(pos, dim: int, base: float) -> np.ndarray:
    """Angle of pair i at each position: pos * base^(-2i/dim), shape pos.shape + (dim/2,)."""
    if dim % 2:
        raise ValueError("RoPE needs an even width")
    i = np.arange(dim // 2, dtype=np.float64)
    inv_freq = np.power(float(base), -2.0 * i / dim)
    return np.asarray(pos, dtype=np.float64)[..., None] * inv_freq


def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate the last axis of x (even width d) pairwise: (x[2i], x[2i+1])
    turned by the angle pos * base^(-2i/d).  pos broadcasts against x's
    leading axes.  fp64 in and out."""
    x = np.asarray(x, dtype=np.float64)
    ang = rope_angles(pos, x.shape[-1], base)
    c, s = np.cos(ang), np.sin(ang)
    even, odd = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = even * c - odd * s
    out[..., 1::2] = even * s + odd * c
    return out


def slot_of(block_table, b: int, pos: int, max_pages_per_seq: int):
    """(page, slot) of cache position pos of sequence b: page block_table[b][pos // 64]
    (page b * max_pages_per_seq + pos // 64 for a contiguous cache), slot pos % 64."""
    i = pos // PAGE
    page = int(block_table[b][i]) if block_table is not None else b * max_pages_per_seq + i
    return page, pos % PAGE


def append_latent(cache: np.ndarray, rows: np.ndarray, pos: np.ndarray, block_table, d_rope: int,
                  base: float | None) -> np.ndarray:
    """Write new token rows into a latent cache (fp64 copy of it returned).

    cache: [num_pages][64][row] (row = num_kv * d_nope + d_rope); rows:
    [B][Q][row], the rope slice (last d_rope entries) not yet rotated; pos:
    [B][Q] cache positions.  The latent part is stored as given; the rope
    slice is rotated at the token's position (base None: stored as given)."""
    cache = np.array(cache, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    mpps = None if block_table is not None else cache.shape[0] // rows.shape[0]
    B, Q, width = rows.shape
    for b in range(B):
        for i in range(Q):
            p = int(pos[b][i])
            page, slot = slot_of(block_table, b, p, mpps)
            r = rows[b, i].copy()
            if base is not None and d_rope:
                r[width - d_rope:] = rope(r[width - d_rope:], p, base)
            cache[page, slot] = r
    return cache


def append_heads(cache: np.ndarray, kv: np.ndarray, pos: np.ndarray, block_table, base: float | None) -> np.ndarray:
    """The same for a GQA/MQA cache [num_pages][2][64][num_kv][D] and new rows
    kv [B][Q][2][num_kv][D]: K (index 0) rotated over the whole head width at
    the token's position (base None: as given), V (index 1) as given."""
    cache = np.array(cache, dtype=np.float64)
    kv = np.asarray(kv, dtype=np.float64)
    B, Q = kv.shape[:2]
    mpps = None if block_table is not None else cache.shape[0] // B
    for b in range(B):
        for i in range(Q):
            p = int(pos[b][i])
            page, slot = slot_of(block_table, b, p, mpps)
            k = kv[b, i, 0]
            cache[page, 0, slot] = rope(k, p, base) if base is not None else k
            cache[page, 1, slot] = kv[b, i, 1]
    return cache


def head_proj(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Per-head projection y[r, h, :] = x[r, h, :] @ w[h] in fp64.

    x: [rows][H][k], w: [H][k][n] -> y: [rows][H][n].  Query absorption is
    head_proj(q^C, W_UK); the up-projection is head_proj(o, W_UV), with the
    R branch outputs of MLRA side by side in o's last axis."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    return np.einsum("rhk,hkn->rhn", x, w)


def materialized_attention(q_c, q_r, latent, k_r, w_uk, w_uv, scale):
    """Decode attention the explicit way (MLA explainer sections 2.2-2.3),
    for one sequence: every head's keys and values are built from the cache
    before attending.

    q_c: [H][R][d_h] semantic query of each head and branch, q_r: [H][R][d_r]
    rotated position query, latent: [L][R][d_c] cached latent (R branches;
    R = 1 for MLA), k_r: [L][d_r] rotated position keys, w_uk:
    [H][R][d_h][d_c], w_uv: [H][R][d_c][d_v].  Branch r of head h has keys
    [W_UK[h,r] c_r ; k^R] against the query [q^C_{h,r} ; q^R_{h,r}] and values
    c_r W_UV[h,r]; the R branch outputs are summed (MLRA page, "moving the sum
    outside").  Returns [H][d_v]."""
    q_c, q_r = np.asarray(q_c, np.float64), np.asarray(q_r, np.float64)
    latent, k_r = np.asarray(latent, np.float64), np.asarray(k_r, np.float64)
    w_uk, w_uv = np.asarray(w_uk, np.float64), np.asarray(w_uv, np.float64)
    H = q_c.shape[0]
    L, R = latent.shape[:2]
    out = np.zeros((H, w_uv.shape[-1]))
    for h in range(H):
        for r in range(R):
            keys = np.concatenate([latent[:, r, :] @ w_uk[h, r].T, k_r], axis=1)   # [L][d_h + d_r]
            vals = latent[:, r, :] @ w_uv[h, r]                                    # [L][d_v]
            s = scale * (keys @ np.concatenate([q_c[h, r], q_r[h, r]]))
            if L:
                p = np.exp(s - s.max())
                out[h] += (p / p.sum()) @ vals
    return out
