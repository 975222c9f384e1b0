"""Seeded input generators (numpy PCG64), shared by the oracle tests and the CUDA path.

Recipe (same for every workload, seed 0 unless stated):
  * weights: ``default_rng(seed)`` draws W_q [d][H*d_h], W_k [d][n_kv*d_h], W_v [d][n_kv*d_h]
    from N(0, 1/d) in that order, then one log-normal(0, 0.5) scale per (query head, pair)
    and one per (KV head, pair), drawn independently; each scale multiplies the two columns
    2k and 2k+1 of its head in W_q (resp. W_k).  This gives heads uneven per-frequency
    energy, the structure the 2-norm pair selection looks for.
  * calibration tokens: ``default_rng([seed, 4])``, X_cal [t_cal][d] ~ N(0, 1).
  * context tokens of sequence b: ``default_rng([seed, 1, b])``, x [L_b][d] ~ N(0, 1);
    any sequence can be regenerated alone.
  * decode tokens: ``default_rng([seed, 2])``, x_dec [B][d] ~ N(0, 1).
  * ragged lengths: ``default_rng([seed, 3])``, integers uniform in [lo, hi].
Token draws are float32 normals (exact in float64).

``cast`` rounds to the workload dtype (round-to-nearest-even) and returns float64
holding the rounded values; ``to_torch`` gives the same values as a torch tensor of
the storage dtype.  Activations of the synthetic MHA layer (q = x W_q, k = x W_k)
are the layer's own forward pass, computed in float64 from cast operands and then
cast, so both sides receive bit-identical activations.
"""

import numpy as np
import torch

from .configs import Workload

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def cast(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to ``dtype`` and return them as float64."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(_TORCH_DTYPE[dtype]).to(torch.float64).numpy()


def to_torch(a: np.ndarray, dtype: str, device="cpu") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(_TORCH_DTYPE[dtype])
    return t.to(device)


def torch_dtype(dtype: str):
    return _TORCH_DTYPE[dtype]


def layer_weights(wl: Workload) -> dict:
    """W_q, W_k, W_v of the synthetic MHA layer, already cast to ``wl.dtype`` (float64 values)."""
    d, H, nkv, dh = wl.hidden, wl.n_heads, wl.n_kv_heads, wl.head_dim
    rng = np.random.default_rng(wl.seed)
    sd = 1.0 / np.sqrt(d)
    W_q = rng.standard_normal((d, H * dh)) * sd
    W_k = rng.standard_normal((d, nkv * dh)) * sd
    W_v = rng.standard_normal((d, nkv * dh)) * sd
    s_q = rng.lognormal(0.0, 0.5, size=(H, dh // 2))
    s_k = rng.lognormal(0.0, 0.5, size=(nkv, dh // 2))
    W_q = W_q.reshape(d, H, dh // 2, 2) * s_q[None, :, :, None]
    W_k = W_k.reshape(d, nkv, dh // 2, 2) * s_k[None, :, :, None]
    return {
        "W_q": cast(W_q.reshape(d, H * dh), wl.dtype),
        "W_k": cast(W_k.reshape(d, nkv * dh), wl.dtype),
        "W_v": cast(W_v, wl.dtype),
    }


def seq_lens(wl: Workload) -> np.ndarray:
    if wl.fixed_lens is not None:
        return np.asarray(wl.fixed_lens, dtype=np.int64)
    if wl.ctx is not None:
        return np.full(wl.batch, wl.ctx, dtype=np.int64)
    lo, hi = wl.ctx_range
    return np.random.default_rng([wl.seed, 3]).integers(lo, hi + 1, size=wl.batch).astype(np.int64)


def _normals(seed_seq, shape) -> np.ndarray:
    return np.random.default_rng(seed_seq).standard_normal(shape, dtype=np.float32).astype(np.float64)


def calib_tokens(wl: Workload) -> np.ndarray:
    return cast(_normals([wl.seed, 4], (wl.t_cal, wl.hidden)), wl.dtype)


def context_tokens(wl: Workload, b: int, length: int) -> np.ndarray:
    """x [length][d] for sequence b (cast values, float64)."""
    return cast(_normals([wl.seed, 1, b], (length, wl.hidden)), wl.dtype)


def decode_tokens(wl: Workload) -> np.ndarray:
    return cast(_normals([wl.seed, 2], (wl.batch, wl.hidden)), wl.dtype)


def project(x: np.ndarray, W: np.ndarray, dtype: str) -> np.ndarray:
    """One linear projection of the synthetic MHA layer, cast to the layer dtype."""
    return cast(x @ W, dtype)


def calib_activations(wl: Workload, weights: dict):
    """q_cal [t_cal][H][d_h], k_cal [t_cal][n_kv][d_h] (unrotated, cast)."""
    X = calib_tokens(wl)
    q = project(X, weights["W_q"], wl.dtype).reshape(wl.t_cal, wl.n_heads, wl.head_dim)
    k = project(X, weights["W_k"], wl.dtype).reshape(wl.t_cal, wl.n_kv_heads, wl.head_dim)
    return q, k


def decode_queries(wl: Workload, weights: dict) -> np.ndarray:
    """q [B][H][d_h]: the new token's query, unrotated, original dim order (cast)."""
    x = decode_tokens(wl)
    return project(x, weights["W_q"], wl.dtype).reshape(wl.batch, wl.n_heads, wl.head_dim)
