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
        if cfg.cache_kind == _lib.MLA_CACHE_INT4_G32:
            self.c_kv = torch.zeros(B, T_cap, cfg.d_c // 2, dtype=torch.uint8, device=device)
            self.c_scales = torch.zeros(B, T_cap, cfg.d_c // 32, dtype=torch.float16, device=device)
        else:
            self.c_kv = torch.zeros(B, T_cap, cfg.d_c, dtype=dt, device=device)
            self.c_scales = None
        R = cfg.n_kv_heads * 2 * cfg.r_pairs
        self.k_rope = torch.zeros(B, T_cap, cfg.n_kv_heads, 2 * cfg.r_pairs, dtype=dt, device=device) \
            if R > 0 else None
        self.struct = _lib.cache_struct(self.c_kv, self.c_scales, self.k_rope, B, T_cap)

    def nbytes_used(self, seq_lens) -> int:
        per_tok = _lib.mla_cache_bytes_per_token(self.cfg)
        return int(sum(int(x) for x in seq_lens)) * per_tok


def workspace(plan: "_lib.Plan", B: int, device="cuda") -> torch.Tensor:
    n = _lib.mla_decode_workspace_bytes(plan, B)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)
