"""Caller-side cache and workspace allocation with torch (device memory plumbing).

The library never allocates inside mla_append/mla_decode: the caller owns the cache
tensors laid out as include/mla_api.h documents and passes an MlaCache view.
"""

import torch

from . import _lib

_DT = {_lib.MLA_F32: torch.float32, _lib.MLA_BF16: torch.bfloat16}


class LatentCache:
    def __init__(self, cfg: "_lib.MlaConfig", B: int, T_cap: int, device="cuda"):
        self.cfg, self.B, self.T_cap = cfg, int(B), int(T_cap)
        dt = _DT[cfg.dtype]
        if cfg.cache_kind in (_lib.MLA_CACHE_INT4_G32, _lib.MLA_CACHE_INT4_G32_R128):
            self.c_kv = torch.zeros(B, T_cap, cfg.d_c // 2, dtype=torch.uint8, device=device)
            self.c_scales = torch.zeros(B, T_cap, cfg.d_c // 32, dtype=torch.float16, device=device)
        else:
            self.c_kv = torch.zeros(B, T_cap, cfg.d_c, dtype=dt, device=device)
            self.c_scales = None
        self.c_resid = self.resid_pos = None
        if cfg.cache_kind == _lib.MLA_CACHE_INT4_G32_R128:
            # the residual ring and the position each slot holds (-1: none yet)
            W = _lib.MLA_RESID_WINDOW
            self.c_resid = torch.zeros(B, W, cfg.d_c, dtype=dt, device=device)
            self.resid_pos = torch.full((B, W), -1, dtype=torch.int32, device=device)
        R = cfg.n_kv_heads * 2 * cfg.r_pairs
        # blocked layout [B][ceil(T_cap/32)][n_kv][32][2r] (see mla_cache_t)
        self.k_rope = torch.zeros(B, (T_cap + 31) // 32, cfg.n_kv_heads, 32, 2 * cfg.r_pairs, dtype=dt,
                                  device=device) if R > 0 else None
        self.struct = _lib.cache_struct(self.c_kv, self.c_scales, self.k_rope, B, T_cap, self.c_resid,
                                        self.resid_pos)

    def reset_sequence(self, b: int) -> None:
        """Forget sequence b's residual window before a new sequence takes slot b."""
        if self.resid_pos is not None:
            self.resid_pos[b].fill_(-1)

    def _kr_index(self, t0: int, t1: int):
        t = torch.arange(t0, t1, device=self.k_rope.device)
        return t // 32, t % 32

    def k_rope_tokens(self, b: int, t0: int, t1: int) -> torch.Tensor:
        """RoPE key dims of tokens [t0, t1) of sequence b, as [t1-t0][n_kv][2r] (a copy)."""
        blk, row = self._kr_index(t0, t1)
        return self.k_rope[b].permute(0, 2, 1, 3)[blk, row]

    def set_k_rope_tokens(self, b: int, t0: int, values: torch.Tensor) -> None:
        """Write [n][n_kv][2r] RoPE key dims as tokens [t0, t0+n) of sequence b."""
        blk, row = self._kr_index(t0, t0 + values.shape[0])
        self.k_rope[b].permute(0, 2, 1, 3)[blk, row] = values.to(self.k_rope.dtype)

    def nbytes_used(self, seq_lens) -> int:
        per_tok = _lib.mla_cache_bytes_per_token(self.cfg)
        return int(sum(int(x) for x in seq_lens)) * per_tok


def workspace(plan: "_lib.Plan", B: int, device="cuda") -> torch.Tensor:
    n = _lib.mla_decode_workspace_bytes(plan, B)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)
