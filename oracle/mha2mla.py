"""Float64 reference of MHA2MLA conversion, latent-cache append and decode.

Test infrastructure only (see package docstring).  Notation: d hidden, H query
heads, n_kv KV heads, G = H / n_kv, g(h) = floor(h / G), d_h head dim, r kept
frequency pairs per KV head, d_c latent width.  Pairs are the 2-D subspaces
(2k, 2k+1), k = 0 .. d_h/2 - 1.

Readings taken where the pages are silent:
  * RoPE: interleaved pairs (2k, 2k+1) as the notes write them; frequency
    theta_k = base^(-2k/d_h); 0-based positions; rotation
    (a, b) -> (a cos p*theta - b sin p*theta, a sin p*theta + b cos p*theta).
  * GQA score aggregation: average of the pair scores over the group's query heads.
  * Top-r tie-break: larger score first, equal scores -> lower pair index.
  * Joint SVD concatenates column blocks (x W maps d -> width), W_dkv = U_trunc and
    Sigma V^T is split per head, literally as the notes state; U column signs are
    normalised (largest-|.| entry positive) for reproducibility only.
  * Softmax scale 1/sqrt(d_h) of the original MHA layer.
  * int4 latent: per token, groups of 32 elements, fp16 scale = fp16(absmax/7),
    code = clamp(round_half_even(c / scale), -7, 7), decided in float32.
"""

import numpy as np

__all__ = [
    "rope_theta", "rotate", "pair_norms", "pair_scores", "select_pairs", "fixed_pairs", "split_dims",
    "svd_joint", "svd_split", "krope_weights", "convert", "append", "quant_int4_g32", "dequant_int4_g32",
    "pack_int4", "unpack_int4", "residual_window", "quant_int2_g32", "dequant_int2_g32", "pack_int2",
    "unpack_int2", "decode_unabsorbed", "decode_absorbed", "decode_sequence",
    "mha_textbook_rope", "cache_bytes_per_token", "mha_cache_bytes_per_token",
]


# --------------------------------------------------------------------------- RoPE
def rope_theta(head_dim: int, base: float) -> np.ndarray:
    """theta_k = base^(-2k/d_h), k = 0..d_h/2-1.

    NOTES §关键设计 / contribution-aware partial-RoPE: RoPE splits q and k into d_h/2
    two-dimensional subspaces, each rotated at its own frequency.  The frequency
    formula is the standard RoPE one (the pages do not print it; base 10000 is the
    workload's stated base).
    """
    k = np.arange(head_dim // 2, dtype=np.float64)
    return base ** (-2.0 * k / head_dim)


def rotate(v: np.ndarray, pos, theta: np.ndarray) -> np.ndarray:
    """Rotate pairs of ``v`` [..., P, 2] by angle pos*theta[P] (pos broadcastable to v[..., 0, 0]).

    NOTES §关键设计: each 2-D subspace [2k, 2k+1] is a rotation at its own frequency.
    """
    pos = np.asarray(pos, dtype=np.float64)
    ang = pos[..., None] * theta  # [..., P]
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[..., 0], v[..., 1]
    return np.stack([a * c - b * s, a * s + b * c], axis=-1)


# ----------------------------------------------------------------- pair selection
def pair_norms(x: np.ndarray) -> np.ndarray:
    """||x^[2k,2k+1]||_2 for every pair: x [..., d_h] -> [..., d_h/2]."""
    xp = x.reshape(*x.shape[:-1], x.shape[-1] // 2, 2)
    return np.sqrt(xp[..., 0] ** 2 + xp[..., 1] ** 2)


def pair_scores(q_cal: np.ndarray, k_cal: np.ndarray) -> np.ndarray:
    """2-norm contribution score per (KV head g, pair k).

    NOTES §关键设计 / contribution-aware partial-RoPE: the contribution of subspace k to
    the attention score is bounded (Cauchy-Schwarz) by ||q^[2k,2k+1]|| * ||k^[2k,2k+1]||;
    the score is that bound averaged over calibration tokens.  Both norms are
    rotation-invariant, so unrotated q/k give the same value.  For GQA the pair set
    is shared by a KV group, so the bound is averaged over the group's query heads.

    q_cal [T][H][d_h], k_cal [T][n_kv][d_h]  ->  contrib [n_kv][d_h/2]
    """
    T, H, dh = q_cal.shape
    n_kv = k_cal.shape[1]
    G = H // n_kv
    qn = pair_norms(q_cal)            # [T][H][P]
    kn = pair_norms(k_cal)            # [T][n_kv][P]
    contrib = np.zeros((n_kv, dh // 2))
    for g in range(n_kv):
        acc = np.zeros(dh // 2)
        for h in range(g * G, (g + 1) * G):
            acc += (qn[:, h, :] * kn[:, g, :]).sum(axis=0)
        contrib[g] = acc / (T * G)
    return contrib


def select_pairs(contrib: np.ndarray, r: int) -> np.ndarray:
    """Head-wise top-r pairs by score, returned ascending per head.

    NOTES §关键设计: keep RoPE on the r subspaces with the largest contribution;
    §关键发现: the selection is head-wise.  Ties: the lower pair index wins.
    """
    n_kv, P = contrib.shape
    out = np.zeros((n_kv, r), dtype=np.int64)
    for g in range(n_kv):
        order = sorted(range(P), key=lambda k: (-contrib[g, k], k))
        out[g] = sorted(order[:r])
    return out


def fixed_pairs(strategy: str, head_dim: int, r: int, n_kv: int) -> np.ndarray:
    """The fixed partial-RoPE pair sets the 2-norm selection is compared against.

    README "MHA2MLA" §Fine-Tuning strategy tables (partial-RoPE versions: full-RoPE,
    S_high, S_uniform, S_2-norm, S_low) and Notes §消融实验 (Partial-RoPE strategy
    comparison: keep high-frequency / low-frequency / uniformly spaced subspaces).  The
    pages give no formulas; the reading: with P = d_h/2 pairs and theta_k = base^(-2k/d_h)
    (pair 0 rotates fastest),
      'high'    the r highest frequencies, k = 0 .. r-1
      'low'     the r lowest frequencies,  k = P-r .. P-1
      'uniform' r pairs evenly spaced from k = 0, k_j = floor(j * P / r)
      'full'    every pair (r = P)
    The same set serves every KV head.  Returns [n_kv][r] int64, ascending.
    """
    P = head_dim // 2
    if not 0 <= r <= P:
        raise ValueError("r out of range")
    if strategy == "high":
        ks = list(range(r))
    elif strategy == "low":
        ks = list(range(P - r, P))
    elif strategy == "uniform":
        ks = [(j * P) // r for j in range(r)]
    elif strategy == "full":
        if r != P:
            raise ValueError("full RoPE keeps every pair")
        ks = list(range(P))
    else:
        raise ValueError(strategy)
    return np.array([ks] * n_kv, dtype=np.int64).reshape(n_kv, r)


def split_dims(pair_idx: np.ndarray, head_dim: int):
    """(rope_dims [n_kv][2r], nope_dims [n_kv][d_h-2r]) for each KV head.

    NOTES §方法详解/整体框架: RoPE is removed from the non-selected subspaces, which
    become NoPE dims.  Rope dims keep ascending-pair order, (2k, 2k+1) adjacent;
    NoPE dims are the ascending complement.
    """
    n_kv, r = pair_idx.shape
    rope = np.zeros((n_kv, 2 * r), dtype=np.int64)
    nope = np.zeros((n_kv, head_dim - 2 * r), dtype=np.int64)
    for g in range(n_kv):
        rd = []
        for k in pair_idx[g]:
            rd += [2 * int(k), 2 * int(k) + 1]
        rope[g] = rd
        nope[g] = [i for i in range(head_dim) if i not in set(rd)]
    return rope, nope


# ------------------------------------------------------------------- joint SVD
def svd_joint(W_k: np.ndarray, W_v: np.ndarray, pair_idx: np.ndarray, d_c: int, head_dim: int):
    """SVDjoint low-rank initialisation.

    NOTES §关键设计 / 联合 SVD 低秩近似 (SVDjoint): concatenate every head's W_k,nope and
    W_v, take a truncated SVD U Sigma V^T, use W_dkv = U_trunc as the down-projection
    producing c_kv, and split Sigma V^T per head into the up-projections W_uk, W_uv.
    The notes print the concatenation's width garbled; it is read as a column
    concatenation [d x (n_kv (d_h-2r) + n_kv d_h)].

    Returns W_dkv [d][d_c], W_uk [n_kv][d_c][d_h-2r], W_uv [n_kv][d_c][d_h], sigma (all).
    """
    n_kv = W_v.shape[1] // head_dim
    _, nope = split_dims(pair_idx, head_dim)
    dn = nope.shape[1]
    blocks = [W_k[:, g * head_dim + nope[g]] for g in range(n_kv)]
    W_kv = np.concatenate(blocks + [W_v], axis=1)
    U, s, Vt = np.linalg.svd(W_kv, full_matrices=False)
    U = U[:, :d_c].copy()
    Vt = Vt[:d_c].copy()
    for i in range(d_c):
        j = int(np.argmax(np.abs(U[:, i])))
        if U[j, i] < 0:
            U[:, i] *= -1.0
            Vt[i] *= -1.0
    M = s[:d_c, None] * Vt
    W_uk = np.stack([M[:, g * dn:(g + 1) * dn] for g in range(n_kv)])
    off = n_kv * dn
    W_uv = np.stack([M[:, off + g * head_dim: off + (g + 1) * head_dim] for g in range(n_kv)])
    return U, W_uk, W_uv, s


def _truncated_svd(W: np.ndarray, rank: int):
    """U[:, :rank], Sigma V^T[:rank] with the sign convention of svd_joint, and all sigmas.
    A rank beyond the matrix's own leaves the extra latent dims empty (zero columns of U
    and zero rows of Sigma V^T)."""
    U, s, Vt = np.linalg.svd(W, full_matrices=False)
    k = min(rank, s.shape[0])
    Uk = np.zeros((W.shape[0], rank))
    M = np.zeros((rank, W.shape[1]))
    Uk[:, :k] = U[:, :k]
    M[:k] = s[:k, None] * Vt[:k]
    for i in range(k):
        j = int(np.argmax(np.abs(Uk[:, i])))
        if Uk[j, i] < 0:
            Uk[:, i] *= -1.0
            M[i] *= -1.0
    return Uk, M, s


def svd_split(W_k: np.ndarray, W_v: np.ndarray, pair_idx: np.ndarray, d_c: int, head_dim: int):
    """SVDsplit low-rank initialisation: separate truncated SVDs of the NoPE key projection
    [W_k,nope(g) for all g] and of W_v.

    README "MHA2MLA" §Fine-Tuning strategy tables (SVD version 2, SVD_split); Notes
    §消融实验 (SVD strategy comparison: SVDsplit and SVDjoint have the same KV cache size).
    Reading: the d_c cached latent dims are split evenly, c = [c_k | c_v] with c_k = x U_k
    (d_c/2 dims) and c_v = x U_v (d_c - d_c/2 dims).  In the shared-latent form used by
    the cache and the decode, W_dkv = [U_k | U_v], W_uk[g] has zero rows for c_v and
    W_uv[g] zero rows for c_k, so K_nope = c_k (Sigma V^T)_k and V = c_v (Sigma V^T)_v.

    Returns W_dkv [d][d_c], W_uk [n_kv][d_c][d_h-2r], W_uv [n_kv][d_c][d_h],
    (sigma_k, sigma_v) (all singular values of each part).
    """
    n_kv = W_v.shape[1] // head_dim
    _, nope = split_dims(pair_idx, head_dim)
    dn = nope.shape[1]
    dk = d_c // 2
    dv = d_c - dk
    Wk_nope = np.concatenate([W_k[:, g * head_dim + nope[g]] for g in range(n_kv)], axis=1)
    U_k, M_k, s_k = _truncated_svd(Wk_nope, dk)
    U_v, M_v, s_v = _truncated_svd(W_v, dv)
    W_dkv = np.concatenate([U_k, U_v], axis=1)
    W_uk = np.zeros((n_kv, d_c, dn))
    W_uv = np.zeros((n_kv, d_c, head_dim))
    for g in range(n_kv):
        W_uk[g, :dk] = M_k[:, g * dn:(g + 1) * dn]
        W_uv[g, dk:] = M_v[:, g * head_dim:(g + 1) * head_dim]
    return W_dkv, W_uk, W_uv, (s_k, s_v)


def krope_weights(W_k: np.ndarray, pair_idx: np.ndarray, head_dim: int) -> np.ndarray:
    """W_krope [d][n_kv][2r]: the columns of W_k that keep RoPE (ascending pair order).

    NOTES §关键设计: the retained subspaces keep their key projection and rotation.
    """
    n_kv = pair_idx.shape[0]
    rope, _ = split_dims(pair_idx, head_dim)
    return np.stack([W_k[:, g * head_dim + rope[g]] for g in range(n_kv)], axis=1)


def convert(weights: dict, q_cal: np.ndarray, k_cal: np.ndarray, wl, cast=None, pair_idx=None,
            svd: str = "joint") -> dict:
    """Partial-RoPE (2-norm top-r, or the given pair set) followed by SVDjoint (NOTES
    §方法详解/整体框架), or SVDsplit when svd == "split".

    ``cast`` (optional) rounds the deployed matrices to the storage dtype; the
    uncast float64 results are kept under '*_exact'.
    """
    contrib = pair_scores(q_cal, k_cal)
    if pair_idx is None:
        pair_idx = select_pairs(contrib, wl.r_pairs)
    low_rank = svd_split if svd == "split" else svd_joint
    W_dkv, W_uk, W_uv, sigma = low_rank(weights["W_k"], weights["W_v"], pair_idx, wl.d_c, wl.head_dim)
    W_kr = krope_weights(weights["W_k"], pair_idx, wl.head_dim)
    out = {"contrib": contrib, "pair_idx": pair_idx, "sigma": sigma,
           "W_dkv_exact": W_dkv, "W_uk_exact": W_uk, "W_uv_exact": W_uv, "W_krope_exact": W_kr}
    c = cast if cast is not None else (lambda a: a)
    out.update(W_dkv=c(W_dkv), W_uk=c(W_uk), W_uv=c(W_uv), W_krope=c(W_kr))
    return out


# ----------------------------------------------------------------------- append
def append(x: np.ndarray, pos: np.ndarray, W_dkv: np.ndarray, W_krope: np.ndarray,
           pair_idx: np.ndarray, theta: np.ndarray):
    """Cache entries of tokens x [N][d] at positions pos [N].

    NOTES §关键设计 / SVDjoint: c_kv = x W_dkv is the cached latent; the retained RoPE
    key dims of each KV head are x W_krope[g], rotated at the token's position with the
    frequencies of that head's kept pairs.

    Returns c [N][d_c], kr [N][n_kv][2r] (float64).
    """
    N = x.shape[0]
    n_kv, r = pair_idx.shape
    c = x @ W_dkv
    kr = np.einsum("nd,dgj->ngj", x, W_krope).reshape(N, n_kv, r, 2)
    th = theta[pair_idx]                                    # [n_kv][r]
    ang = np.asarray(pos, dtype=np.float64)[:, None, None] * th[None]
    cs, sn = np.cos(ang), np.sin(ang)
    a, b = kr[..., 0], kr[..., 1]
    kr = np.stack([a * cs - b * sn, a * sn + b * cs], axis=-1).reshape(N, n_kv, 2 * r)
    return c, kr


# ------------------------------------------------------------------------- int4
def quant_int4_g32(c: np.ndarray):
    """Per-token int4 quantisation of the latent in groups of 32.

    NOTES §关键设计 / KV-cache quantisation: the latent c_kv is a standard MLA latent
    and 4-bit quantisation stacks on it.  The encoding is a reading (the pages name
    4-bit, the official evaluation uses an HQQ backend): symmetric, scale fp16(absmax/7),
    code clamp(rint_half_even(c/scale), -7, 7); an all-zero group (or a scale that
    rounds to 0) gives scale 0 and codes 0.  Decisions are taken in float32, the
    precision in which the latent is produced.

    c [N][d_c] -> codes int8 [N][d_c], scales float16 [N][d_c/32]
    """
    c32 = np.asarray(c, dtype=np.float64).astype(np.float32)
    N, dc = c32.shape
    g = c32.reshape(N, dc // 32, 32)
    absmax = np.abs(g).max(axis=-1)                                   # float32, exact
    scale16 = (absmax / np.float32(7.0)).astype(np.float32).astype(np.float16)
    sc32 = scale16.astype(np.float32)
    safe = np.where(sc32 > 0, sc32, np.float32(1.0))
    q = np.rint((g / safe[..., None]).astype(np.float32))
    q = np.clip(q, -7, 7)
    q = np.where(sc32[..., None] > 0, q, 0)
    return q.astype(np.int8).reshape(N, dc), scale16


def dequant_int4_g32(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """value = code * scale (exact in float64)."""
    N, dc = codes.shape
    return (codes.reshape(N, dc // 32, 32).astype(np.float64)
            * scales.astype(np.float64)[..., None]).reshape(N, dc)


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Two's-complement nibbles, element 2i in the low nibble of byte i."""
    u = (codes.astype(np.int16) & 0xF).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    lo = (packed & 0xF).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def quant_int2_g32(c: np.ndarray):
    """Per-token 2-bit quantisation of the latent in groups of 32.

    NOTES §关键设计 / KV-cache quantisation: 4-bit or 2-bit quantisation stacks on the
    latent.  The reading is the int4 encoding's scheme at 2 bits: symmetric, zero is a
    level, codes clamp(rint_half_even(c/scale), -1, 1) (the largest magnitude 2^(2-1)-1),
    scale fp16(absmax / 1); an all-zero group (or a scale that rounds to 0) gives scale 0
    and codes 0.  Decisions are taken in float32.

    c [N][d_c] -> codes int8 [N][d_c] in {-1, 0, 1}, scales float16 [N][d_c/32]
    """
    c32 = np.asarray(c, dtype=np.float64).astype(np.float32)
    N, dc = c32.shape
    g = c32.reshape(N, dc // 32, 32)
    scale16 = np.abs(g).max(axis=-1).astype(np.float16)
    sc32 = scale16.astype(np.float32)
    safe = np.where(sc32 > 0, sc32, np.float32(1.0))
    q = np.clip(np.rint((g / safe[..., None]).astype(np.float32)), -1, 1)
    q = np.where(sc32[..., None] > 0, q, 0)
    return q.astype(np.int8).reshape(N, dc), scale16


def dequant_int2_g32(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """value = code * scale (exact in float64)."""
    return dequant_int4_g32(codes, scales)


def pack_int2(codes: np.ndarray) -> np.ndarray:
    """Two's-complement 2-bit fields, element 4i + k in bits 2k, 2k+1 of byte i."""
    u = (codes.astype(np.int16) & 0x3).astype(np.uint8)
    return (u[:, 0::4] | (u[:, 1::4] << 2) | (u[:, 2::4] << 4) | (u[:, 3::4] << 6)).astype(np.uint8)


def unpack_int2(packed: np.ndarray) -> np.ndarray:
    out = np.empty((packed.shape[0], packed.shape[1] * 4), dtype=np.int8)
    for k in range(4):
        f = ((packed >> (2 * k)) & 0x3).astype(np.int16)
        out[:, k::4] = np.where(f >= 2, f - 4, f)
    return out


def residual_window(c_quant: np.ndarray, c_plain: np.ndarray, window: int) -> np.ndarray:
    """Latent values a decode reads from the int4 cache with an unquantised residual window.

    README "MHA2MLA" (LongBench evaluation of the 4-bit quantised cache) runs the cache with
    a residual length of 128; the reading taken here: the `window` most recent tokens are
    read with their unquantised value (as stored, in the cache dtype) and every older token
    with its int4 value.  Tokens are appended in position order, so for a sequence of L
    tokens the window is rows [max(0, L - window), L).

    c_quant, c_plain [L][d_c] -> [L][d_c] (float64)
    """
    c_quant = np.asarray(c_quant, dtype=np.float64)
    c_plain = np.asarray(c_plain, dtype=np.float64)
    assert c_quant.shape == c_plain.shape and window >= 0
    L = c_quant.shape[0]
    out = c_quant.copy()
    lo = max(0, L - window)
    out[lo:] = c_plain[lo:]
    return out


# ----------------------------------------------------------------------- decode
def _softmax(s: np.ndarray) -> np.ndarray:
    e = np.exp(s - s.max())
    return e / e.sum()


def decode_unabsorbed(q: np.ndarray, c: np.ndarray, kr: np.ndarray, W_uk: np.ndarray,
                      W_uv: np.ndarray, pair_idx: np.ndarray, theta: np.ndarray, scale=None) -> np.ndarray:
    """Attention of one sequence's new query over its latent cache, by definition.

    NOTES §关键设计 / SVDjoint: keys' NoPE part is reconstructed as K_nope = c_kv W_uk and
    values as V = c_kv W_uv; the retained RoPE dims give a separate score term.  The
    query is split the same way: NoPE dims unrotated, kept pairs rotated at the query
    position p = L - 1.  Scale 1/sqrt(d_h), the original layer's, unless `scale` is given
    (a caller-chosen softmax scale multiplies the scores in its place).

    q [H][d_h]; c [L][d_c]; kr [L][n_kv][2r] (already rotated)  ->  o [H][d_h]
    """
    sc = 1.0 / np.sqrt(q.shape[1]) if scale is None else float(scale)
    H, dh = q.shape
    n_kv, r = pair_idx.shape
    G = H // n_kv
    L = c.shape[0]
    p = L - 1
    rope, nope = split_dims(pair_idx, dh)
    th = theta[pair_idx]
    o = np.zeros((H, dh))
    for h in range(H):
        g = h // G
        K_nope = c @ W_uk[g]                      # [L][d_h-2r]
        V = c @ W_uv[g]                           # [L][d_h]
        q_nope = q[h, nope[g]]
        q_rope = rotate(q[h, rope[g]].reshape(r, 2), p, th[g]).reshape(2 * r)
        s = (K_nope @ q_nope + kr[:, g, :] @ q_rope) * sc
        o[h] = _softmax(s) @ V
    return o


def decode_absorbed(q: np.ndarray, c: np.ndarray, kr: np.ndarray, W_uk: np.ndarray,
                    W_uv: np.ndarray, pair_idx: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """The same attention with W_uk absorbed into the query and W_uv applied after the sum.

    NOTES §关键设计 (design motivation): MLA separates RoPE and non-RoPE dims because the
    RoPE part cannot take part in the matrix merge and is computed independently; the
    NoPE part scores against c_kv through q_nope W_uk^T.
    """
    H, dh = q.shape
    n_kv, r = pair_idx.shape
    G = H // n_kv
    L = c.shape[0]
    p = L - 1
    rope, nope = split_dims(pair_idx, dh)
    th = theta[pair_idx]
    o = np.zeros((H, dh))
    for h in range(H):
        g = h // G
        q_lat = W_uk[g] @ q[h, nope[g]]           # [d_c]
        q_rope = rotate(q[h, rope[g]].reshape(r, 2), p, th[g]).reshape(2 * r)
        s = (c @ q_lat + kr[:, g, :] @ q_rope) / np.sqrt(dh)
        O_lat = _softmax(s) @ c                   # [d_c]
        o[h] = O_lat @ W_uv[g]
    return o


def decode_sequence(q, c, kr, conv: dict, theta, absorbed=False):
    f = decode_absorbed if absorbed else decode_unabsorbed
    return f(q, c, kr, conv["W_uk"], conv["W_uv"], conv["pair_idx"], theta)


# --------------------------------------------------------- textbook MHA (pin only)
def mha_textbook_rope(q: np.ndarray, k: np.ndarray, v: np.ndarray, theta: np.ndarray,
                      rope_pairs=None) -> np.ndarray:
    """Plain GQA/MHA decode with (partial) RoPE, written with explicit loops.

    q [H][d_h] at position L-1; k, v [L][n_kv][d_h] unrotated.  ``rope_pairs[g]`` is
    the set of pairs rotated for KV group g (None: all pairs; empty: NoPE).  Used only
    to pin the converted form against the original layer (full-rank latent).
    """
    H, dh = q.shape
    L, n_kv, _ = k.shape
    G = H // n_kv
    o = np.zeros((H, dh))
    for h in range(H):
        g = h // G
        rot = set(range(dh // 2)) if rope_pairs is None else set(int(x) for x in rope_pairs[g])
        qr = q[h].copy()
        for kk in range(dh // 2):
            if kk in rot:
                a, b = q[h, 2 * kk], q[h, 2 * kk + 1]
                ang = (L - 1) * theta[kk]
                qr[2 * kk] = a * np.cos(ang) - b * np.sin(ang)
                qr[2 * kk + 1] = a * np.sin(ang) + b * np.cos(ang)
        s = np.zeros(L)
        for t in range(L):
            kt = k[t, g].copy()
            for kk in range(dh // 2):
                if kk in rot:
                    a, b = k[t, g, 2 * kk], k[t, g, 2 * kk + 1]
                    ang = t * theta[kk]
                    kt[2 * kk] = a * np.cos(ang) - b * np.sin(ang)
                    kt[2 * kk + 1] = a * np.sin(ang) + b * np.cos(ang)
            s[t] = float(np.dot(qr, kt)) / np.sqrt(dh)
        w = np.exp(s - s.max())
        w /= w.sum()
        for t in range(L):
            o[h] += w[t] * v[t, g]
    return o


# ------------------------------------------------------------------- accounting
def cache_bytes_per_token(n_kv: int, r: int, d_c: int, elem_bytes: int, int4: bool = False,
                          count_scales: bool = True) -> float:
    """Bytes cached per token per layer.

    NOTES §关键设计 (SVDjoint and the KV-cache quantisation paragraph): the cache holds
    the latent c_kv plus each KV head's 2r retained RoPE key dims; with 4-bit
    quantisation the latent is stored at 4 bits per element (plus one fp16 scale per
    32 elements when ``count_scales``), the RoPE dims stay in the storage dtype.
    """
    rope = n_kv * 2 * r * elem_bytes
    if not int4:
        return d_c * elem_bytes + rope
    lat = d_c / 2.0 + (2.0 * d_c / 32.0 if count_scales else 0.0)
    return lat + rope


def mha_cache_bytes_per_token(n_kv: int, head_dim: int, elem_bytes: int) -> int:
    """Full K and V per token per layer: 2 n_kv d_h elements (NOTES §研究背景与动机)."""
    return 2 * n_kv * head_dim * elem_bytes
