"""Shared set-up for the parity tests: the oracle's side of every comparison.

Only the tests use this module.  It calls the oracle and the seeded generators; the
CUDA path is exercised separately by each test through the C-ABI binding.
"""

import numpy as np
import torch

import oracle as O
from workloads import generate as gen

# tolerances (float configs: rel-L2; bf16/int4: rel-L2 and max-abs)
TOL_F32_REL = 1e-5
TOL_BF16_REL = 1e-2
TOL_BF16_ABS = 3e-2


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_close(got, ref, dtype: str, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rl = rel_l2(got, ref)
    if dtype == "f32":
        assert rl <= TOL_F32_REL, f"{what}: rel-L2 {rl:.3e} > {TOL_F32_REL}"
    else:
        ma = float(np.max(np.abs(got - ref))) if got.size else 0.0
        assert rl <= TOL_BF16_REL and ma <= TOL_BF16_ABS, f"{what}: rel-L2 {rl:.3e}, max-abs {ma:.3e}"
    return rl


def bf16_ulp(x):
    """Spacing of bfloat16 numbers at |x| (8 significand bits)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_stored_close(got, exact, dtype: str, what: str = ""):
    """Cache entries are stored in the config dtype, so they are compared with the exact
    float64 value within one unit in the last place of that dtype (the kernel rounds a
    float32 sum once; when the sum sits next to a rounding midpoint it may land on the
    other neighbour), plus the rel-L2 bound.  A fixed 3e-2 absolute bound is below the
    bf16 spacing for |x| >= 8, so it cannot apply to stored values."""
    got = np.asarray(got, dtype=np.float64)
    exact = np.asarray(exact, dtype=np.float64)
    assert got.shape == exact.shape and np.all(np.isfinite(got)), what
    rl = rel_l2(got, exact)
    if dtype == "f32":
        assert rl <= TOL_F32_REL, f"{what}: rel-L2 {rl:.3e}"
        return rl
    err = np.abs(got - exact)
    bound = bf16_ulp(exact) + 1e-6
    worst = float(np.max(err / bound)) if err.size else 0.0
    assert rl <= TOL_BF16_REL and worst <= 1.0, f"{what}: rel-L2 {rl:.3e}, worst error {worst:.2f} ulp"
    return rl


def quant_scheme(wl):
    """(quantise, dequantise, pack, unpack) of the workload's quantised latent cache, or None."""
    if wl.cache == "int4_g32":
        return O.quant_int4_g32, O.dequant_int4_g32, O.pack_int4, O.unpack_int4
    if wl.cache == "int2_g32":
        return O.quant_int2_g32, O.dequant_int2_g32, O.pack_int2, O.unpack_int2
    return None


class OracleCase:
    """Oracle conversion, cache and reference outputs for one workload (float64)."""

    def __init__(self, wl, seqs=None, pairs=None, svd="joint"):
        """pairs: None for the 2-norm selection, else a fixed strategy name of
        oracle.fixed_pairs ('high', 'low', 'uniform', 'full'); svd: 'joint' or 'split'."""
        self.wl = wl
        self.w = gen.layer_weights(wl)
        self.q_cal, self.k_cal = gen.calib_activations(wl, self.w)
        cast = lambda a: gen.cast(a, wl.dtype)  # noqa: E731
        pair_idx = None if pairs is None else O.fixed_pairs(pairs, wl.head_dim, wl.r_pairs, wl.n_kv_heads)
        self.conv = O.convert(self.w, self.q_cal, self.k_cal, wl, cast=cast, pair_idx=pair_idx, svd=svd)
        self.theta = O.rope_theta(wl.head_dim, wl.rope_base)
        self.lens = gen.seq_lens(wl)
        self.q = gen.decode_queries(wl, self.w)
        self.x_dec = gen.decode_tokens(wl)
        self.seqs = list(range(wl.batch)) if seqs is None else list(seqs)
        self.cache = {}
        for b in self.seqs:
            self.cache[b] = self._sequence_cache(b)

    def tokens(self, b):
        """x [L_b][d]: context tokens at 0..L-2 and the decode token at L-1."""
        L = int(self.lens[b])
        if L == 0:
            return np.zeros((0, self.wl.hidden))
        ctx = gen.context_tokens(self.wl, b, L - 1)
        return np.concatenate([ctx, self.x_dec[b:b + 1]], axis=0)

    def _sequence_cache(self, b):
        wl, cv = self.wl, self.conv
        x = self.tokens(b)
        L = x.shape[0]
        c, kr = O.append(x, np.arange(L), cv["W_dkv"], cv["W_krope"], cv["pair_idx"], self.theta)
        out = {"c_exact": c, "kr_exact": kr, "kr": gen.cast(kr, wl.dtype)}
        qs = quant_scheme(wl)
        if qs is not None:
            codes, scales = qs[0](c)
            deq = qs[1](codes, scales)
            out.update(codes=codes, scales=scales, c=deq)
            if wl.resid:   # the most recent tokens are read unquantised, as stored (dtype)
                out["c"] = O.residual_window(deq, gen.cast(c, wl.dtype), wl.resid)
        else:
            out["c"] = gen.cast(c, wl.dtype)
        return out

    def reference(self, b, h=None):
        """Oracle decode of sequence b over its stored cache values -> [H][d_h] (or [d_h])."""
        L = int(self.lens[b])
        if L == 0:
            o = np.zeros((self.wl.n_heads, self.wl.head_dim))
        else:
            cc = self.cache[b]
            o = O.decode_unabsorbed(self.q[b], cc["c"], cc["kr"], self.conv["W_uk"], self.conv["W_uv"],
                                    self.conv["pair_idx"], self.theta)
        return o if h is None else o[h]


def t_dtype(wl):
    return gen.torch_dtype(wl.dtype)


def upload_oracle_cache(case: OracleCase, cache, T_cap):
    """Write the oracle's stored cache values into a LatentCache (host -> device copies)."""
    wl = case.wl
    for b in case.seqs:
        L = int(case.lens[b])
        if L == 0:
            continue
        cc = case.cache[b]
        qs = quant_scheme(wl)
        if qs is not None:
            cache.set_latent_rows(b, 0, torch.from_numpy(qs[2](cc["codes"])))
            cache.set_scale_rows(b, 0, torch.from_numpy(cc["scales"]))
            if wl.resid:   # ring slot t % W holds token t for the window's tokens
                W = cache.c_resid.shape[1]
                t = np.arange(max(0, L - W), L)
                cache.c_resid[b, t % W] = gen.to_torch(cc["c_exact"][t], wl.dtype, cache.c_resid.device)
                cache.resid_pos[b, t % W] = torch.from_numpy(t.astype(np.int32)).to(cache.resid_pos.device)
        else:
            cache.set_latent_rows(b, 0, gen.to_torch(cc["c"], wl.dtype, cache.c_kv.device))
        if cache.k_rope is not None:
            cache.set_k_rope_tokens(b, 0, gen.to_torch(cc["kr"], wl.dtype, cache.k_rope.device))


def plan_inputs(case: OracleCase):
    """The oracle's converted weights as host torch tensors for mla_plan_create."""
    wl = case.wl
    cv = case.conv
    td = lambda a: gen.to_torch(a, wl.dtype).contiguous()  # noqa: E731
    return dict(W_dkv=td(cv["W_dkv"]), W_k=td(case.w["W_k"]),
                pair_idx=torch.from_numpy(np.ascontiguousarray(cv["pair_idx"], dtype=np.int32)),
                W_uk=td(cv["W_uk"]), W_uv=td(cv["W_uv"]))
