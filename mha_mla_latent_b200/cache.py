"""Caller-side cache and workspace allocation with torch (device memory plumbing).

The library never allocates inside mla_append/mla_decode: the caller owns the cache
tensors laid out as include/mla_api.h documents and passes an MlaCache view.
"""

import torch

from . import _lib

_DT = {_lib.MLA_F32: torch.float32, _lib.MLA_BF16: torch.bfloat16}


class LatentCache:
    """The cache arrays of mla_cache_t.  Contiguous by default; with `block_table`
    ([B][T_cap/128] int32 pool block ids, T_cap a multiple of 128) and `n_blocks`, the
    arrays are a pool of 128-token blocks and token t of sequence b lives in block
    block_table[b][t // 128]."""

    def __init__(self, cfg: "_lib.MlaConfig", B: int, T_cap: int, device="cuda", block_table=None,
                 n_blocks: int = 0):
        self.cfg, self.B, self.T_cap = cfg, int(B), int(T_cap)
        dt = _DT[cfg.dtype]
        self.paged = block_table is not None
        if self.paged:
            BT = _lib.MLA_BLOCK_TOKENS
            if T_cap % BT or n_blocks <= 0:
                raise ValueError(f"a paged cache needs T_cap a multiple of {BT} and n_blocks > 0")
            self.block_table = torch.as_tensor(block_table, dtype=torch.int32).to(device).contiguous()
            assert tuple(self.block_table.shape) == (B, T_cap // BT)
            self._table = self.block_table.cpu().numpy()
            self.n_blocks = int(n_blocks)
            rows, cap = self.n_blocks, BT
        else:
            self.block_table, self.n_blocks = None, 0
            rows, cap = B, T_cap
        if cfg.cache_kind in (_lib.MLA_CACHE_INT4_G32, _lib.MLA_CACHE_INT4_G32_R128, _lib.MLA_CACHE_INT2_G32):
            per_byte = 4 if cfg.cache_kind == _lib.MLA_CACHE_INT2_G32 else 2   # codes per byte
            self.c_kv = torch.zeros(rows, cap, cfg.d_c // per_byte, dtype=torch.uint8, device=device)
            self.c_scales = torch.zeros(rows, cap, cfg.d_c // 32, dtype=torch.float16, device=device)
        else:
            self.c_kv = torch.zeros(rows, cap, cfg.d_c, dtype=dt, device=device)
            self.c_scales = None
        self.c_resid = self.resid_pos = None
        if cfg.cache_kind == _lib.MLA_CACHE_INT4_G32_R128:
            # the residual ring and the position each slot holds (-1: none yet)
            W = _lib.MLA_RESID_WINDOW
            self.c_resid = torch.zeros(B, W, cfg.d_c, dtype=dt, device=device)
            self.resid_pos = torch.full((B, W), -1, dtype=torch.int32, device=device)
        R = cfg.n_kv_heads * 2 * cfg.r_pairs
        # token-major layout [B][T_cap][n_kv][2r] (see mla_cache_t; pool blocks when paged)
        self.k_rope = torch.zeros(rows, cap, cfg.n_kv_heads, 2 * cfg.r_pairs, dtype=dt,
                                  device=device) if R > 0 else None
        self.struct = _lib.cache_struct(self.c_kv, self.c_scales, self.k_rope, B, T_cap, self.c_resid,
                                        self.resid_pos, self.block_table, self.n_blocks)

    def _loc(self, b: int, t0: int, t1: int):
        """Storage (row-space sequence, token) of tokens [t0, t1) of sequence b."""
        t = torch.arange(t0, t1)
        if not self.paged:
            return torch.full_like(t, b), t
        BT = _lib.MLA_BLOCK_TOKENS
        return torch.from_numpy(self._table[b])[t // BT].long(), t % BT

    def _rows(self, arr, b, t0, t1):
        pb, pt = self._loc(b, t0, t1)
        return arr[pb.to(arr.device), pt.to(arr.device)]

    def _set_rows(self, arr, b, t0, values):
        pb, pt = self._loc(b, t0, t0 + values.shape[0])
        arr[pb.to(arr.device), pt.to(arr.device)] = values.to(arr.device, arr.dtype)

    def latent_rows(self, b: int, t0: int, t1: int) -> torch.Tensor:
        """c_kv rows of tokens [t0, t1) of sequence b (codes for the int4 cache), a copy."""
        return self._rows(self.c_kv, b, t0, t1)

    def scale_rows(self, b: int, t0: int, t1: int) -> torch.Tensor:
        return self._rows(self.c_scales, b, t0, t1)

    def set_latent_rows(self, b: int, t0: int, values: torch.Tensor) -> None:
        self._set_rows(self.c_kv, b, t0, values)

    def set_scale_rows(self, b: int, t0: int, values: torch.Tensor) -> None:
        self._set_rows(self.c_scales, b, t0, values)

    def query_view(self, seq_of_query) -> "_lib.MlaCache":
        """A cache view with one row per query: query j reads sequence seq_of_query[j]'s blocks.

        Many queries of one sequence (a chunk of new tokens, or drafted tokens to verify)
        then attend causally in a single mla_decode: query j at position p_j is passed with
        seq_lens[j] = p_j + 1, so it is rotated at p_j and attends over tokens [0, p_j].
        Needs the paged layout (the table rows alias the sequence's blocks) and no residual
        window (the ring belongs to a sequence row).  The view holds its own table; keep the
        returned object alive while the call runs."""
        if not self.paged or self.c_resid is not None:
            raise ValueError("query_view needs a paged cache without a residual window")
        idx = torch.as_tensor(seq_of_query, dtype=torch.long)
        table = self.block_table[idx.to(self.block_table.device)].contiguous()
        view = _lib.cache_struct(self.c_kv, self.c_scales, self.k_rope, len(idx), self.T_cap,
                                 block_table=table, n_blocks=self.n_blocks)
        view._table_ref = table   # the struct holds a raw pointer
        return view

    def reset_sequence(self, b: int) -> None:
        """Forget sequence b's residual window before a new sequence takes slot b."""
        if self.resid_pos is not None:
            self.resid_pos[b].fill_(-1)

    def k_rope_tokens(self, b: int, t0: int, t1: int) -> torch.Tensor:
        """RoPE key dims of tokens [t0, t1) of sequence b, as [t1-t0][n_kv][2r] (a copy)."""
        return self._rows(self.k_rope, b, t0, t1)

    def set_k_rope_tokens(self, b: int, t0: int, values: torch.Tensor) -> None:
        """Write [n][n_kv][2r] RoPE key dims as tokens [t0, t0+n) of sequence b."""
        self._set_rows(self.k_rope, b, t0, values)

    def nbytes_used(self, seq_lens) -> int:
        per_tok = _lib.mla_cache_bytes_per_token(self.cfg)
        return int(sum(int(x) for x in seq_lens)) * per_tok


def workspace(plan: "_lib.Plan", B: int, device="cuda") -> torch.Tensor:
    n = _lib.mla_decode_workspace_bytes(plan, B)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)
