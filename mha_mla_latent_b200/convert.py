"""Conversion of an MHA layer into the MLA form the decode library consumes.

Conversion runs once per model, before any decode step:
  1. partial-RoPE pair selection — the library's `mla_select_pairs` kernel (2-norm
     contribution scores, head-wise top-r; paper notes "MHA2MLA" (ACL 2025),
     §关键设计, contribution-aware partial-RoPE removal);
  2. SVDjoint — a truncated SVD of the concatenated NoPE key and value projections
     (§关键设计, 联合 SVD 低秩近似): W_dkv = U_trunc, Sigma V^T split into W_uk, W_uv.
     This is a one-off dense factorisation done with the CUDA solver library through
     torch.linalg.svd in float64 on the device; it is not part of the decode path.
  3. the results are cast to the storage dtype and handed to `mla_plan_create`.
"""

import torch

from . import _lib

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def select_pairs(cfg: "_lib.MlaConfig", q_cal: torch.Tensor, k_cal: torch.Tensor):
    """q_cal [T][H][d_h], k_cal [T][n_kv][d_h] device tensors -> (pair_idx int32 [n_kv][r], contrib)."""
    dev = q_cal.device
    pair_idx = torch.empty(cfg.n_kv_heads, max(cfg.r_pairs, 1), dtype=torch.int32, device=dev)
    contrib = torch.empty(cfg.n_kv_heads, cfg.head_dim // 2, dtype=torch.float32, device=dev)
    _lib.mla_select_pairs(cfg, q_cal.contiguous(), k_cal.contiguous(), pair_idx, contrib)
    return pair_idx[:, :cfg.r_pairs], contrib


def svd_joint(W_k: torch.Tensor, W_v: torch.Tensor, pair_idx: torch.Tensor, d_c: int, head_dim: int):
    """Joint truncated SVD of [W_k,nope(g) for all g | W_v] (float64, on W_k's device)."""
    n_kv = W_v.shape[1] // head_dim
    r = pair_idx.shape[1]
    Wk = W_k.to(torch.float64)
    Wv = W_v.to(torch.float64)
    pidx = pair_idx.to("cpu").tolist()
    blocks = []
    for g in range(n_kv):
        rope = set()
        for k in pidx[g]:
            rope.update((2 * k, 2 * k + 1))
        nope = [i for i in range(head_dim) if i not in rope]
        blocks.append(Wk[:, [g * head_dim + i for i in nope]])
    W_kv = torch.cat(blocks + [Wv], dim=1)
    U, S, Vh = torch.linalg.svd(W_kv, full_matrices=False)
    U, Vh = U[:, :d_c], Vh[:d_c]
    # sign convention: the largest-magnitude entry of each U column is positive
    idx = U.abs().argmax(dim=0)
    sgn = torch.sign(U[idx, torch.arange(d_c, device=U.device)])
    sgn[sgn == 0] = 1.0
    U = U * sgn
    M = (S[:d_c, None] * Vh) * sgn[:, None]
    dn = head_dim - 2 * r
    W_uk = torch.stack([M[:, g * dn:(g + 1) * dn] for g in range(n_kv)])
    off = n_kv * dn
    W_uv = torch.stack([M[:, off + g * head_dim: off + (g + 1) * head_dim] for g in range(n_kv)])
    return U, W_uk, W_uv


def _truncated_svd(W: torch.Tensor, rank: int):
    """U[:, :rank] and Sigma V^T[:rank] (float64) with the sign convention of svd_joint; a
    rank beyond the matrix's own leaves the extra latent dims empty (zeros)."""
    U, S, Vh = torch.linalg.svd(W, full_matrices=False)
    k = min(rank, S.shape[0])
    U, Vh = U[:, :k], Vh[:k]
    idx = U.abs().argmax(dim=0)
    sgn = torch.sign(U[idx, torch.arange(k, device=U.device)])
    sgn[sgn == 0] = 1.0
    Uk = torch.zeros(W.shape[0], rank, dtype=W.dtype, device=W.device)
    M = torch.zeros(rank, W.shape[1], dtype=W.dtype, device=W.device)
    Uk[:, :k] = U * sgn
    M[:k] = (S[:k, None] * Vh) * sgn[:, None]
    return Uk, M


def svd_split(W_k: torch.Tensor, W_v: torch.Tensor, pair_idx: torch.Tensor, d_c: int, head_dim: int):
    """SVD_split (README §Fine-Tuning, SVD version 2): separate truncated SVDs of the NoPE
    key projection and of W_v, d_c/2 latent dims each, in the shared-latent form the cache
    and the decode use: W_dkv = [U_k | U_v], W_uk rows of the c_v half and W_uv rows of the
    c_k half are zero."""
    n_kv = W_v.shape[1] // head_dim
    r = pair_idx.shape[1]
    dn = head_dim - 2 * r
    dk = d_c // 2
    dv = d_c - dk
    Wk = W_k.to(torch.float64)
    pidx = pair_idx.to("cpu").tolist()
    blocks = []
    for g in range(n_kv):
        rope = set()
        for k in pidx[g]:
            rope.update((2 * k, 2 * k + 1))
        blocks.append(Wk[:, [g * head_dim + i for i in range(head_dim) if i not in rope]])
    U_k, M_k = _truncated_svd(torch.cat(blocks, dim=1), dk)
    U_v, M_v = _truncated_svd(W_v.to(torch.float64), dv)
    W_dkv = torch.cat([U_k, U_v], dim=1)
    W_uk = torch.zeros(n_kv, d_c, dn, dtype=torch.float64, device=W_k.device)
    W_uv = torch.zeros(n_kv, d_c, head_dim, dtype=torch.float64, device=W_k.device)
    for g in range(n_kv):
        W_uk[g, :dk] = M_k[:, g * dn:(g + 1) * dn]
        W_uv[g, dk:] = M_v[:, g * head_dim:(g + 1) * head_dim]
    return W_dkv, W_uk, W_uv


def convert_layer(cfg: "_lib.MlaConfig", W_k: torch.Tensor, W_v: torch.Tensor,
                  q_cal: torch.Tensor, k_cal: torch.Tensor, svd: str = "joint") -> dict:
    """Full conversion; returns host tensors in the storage dtype ready for mla_plan_create.
    svd: "joint" (SVDjoint) or "split" (SVD_split)."""
    dtype = "bf16" if cfg.dtype == _lib.MLA_BF16 else "f32"
    tdt = _DT[dtype]
    pair_idx, contrib = select_pairs(cfg, q_cal, k_cal)
    low_rank = svd_split if svd == "split" else svd_joint
    W_dkv, W_uk, W_uv = low_rank(W_k, W_v, pair_idx, cfg.d_c, cfg.head_dim)
    host = lambda t: t.to(tdt).contiguous().cpu()  # noqa: E731
    return {
        "pair_idx": pair_idx.to(torch.int32).contiguous().cpu(),
        "contrib": contrib.cpu(),
        "W_dkv": host(W_dkv),
        "W_k": host(W_k),
        "W_uk": host(W_uk),
        "W_uv": host(W_uv),
    }


def plan_from_converted(cfg: "_lib.MlaConfig", conv: dict) -> "_lib.Plan":
    return _lib.mla_plan_create(cfg, conv["W_dkv"], conv["W_k"], conv["pair_idx"], conv["W_uk"],
                                conv["W_uv"])
