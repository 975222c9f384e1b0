"""ctypes binding of the C ABI in include/mla_api.h.

Argument marshalling only: torch tensors supply device pointers and the current
stream; every computation happens in the CUDA library.  Importing this module
loads the in-tree shared library and fails loudly when it is missing.
"""

import ctypes
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MLA_B200_LIB", os.path.join(_PKG, "lib", "libmla_b200.so"))

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_ALIGNMENT = 0, 1, 2, 3
MLA_ERR_WORKSPACE_TOO_SMALL, MLA_ERR_CUDA, MLA_ERR_DEVICE = 4, 5, 6
MLA_F32, MLA_BF16 = 0, 1
MLA_CACHE_SAME, MLA_CACHE_INT4_G32, MLA_CACHE_INT4_G32_R128, MLA_CACHE_INT2_G32 = 0, 1, 2, 3
MLA_RESID_WINDOW = 128
MLA_OPT_DECODE_KERNEL, MLA_OPT_DECODE_SPLITS, MLA_OPT_PROFILE_EVENTS, MLA_OPT_OVERLAP_LAUNCH = 1, 2, 3, 4
MLA_OPT_WAIT_LIMIT_US, MLA_OPT_TEST_SKIP_COPY, MLA_OPT_PROFILE_KERNELS = 5, 6, 8
MLA_DEVERR_SEQ_LEN, MLA_DEVERR_APPEND_SLOT, MLA_DEVERR_TIMEOUT, MLA_DEVERR_BLOCK = 1, 2, 4, 8
MLA_BLOCK_TOKENS = 128

EXPORTED = (
    "mla_status_string", "mla_version", "mla_cache_bytes_per_token", "mla_select_pairs",
    "mla_plan_create", "mla_plan_destroy", "mla_plan_set_option", "mla_append",
    "mla_decode_workspace_bytes", "mla_decode", "mla_device_error", "mla_decode_noalloc",
    "mla_fixed_pairs", "mla_decode_step", "mla_decode_step_host", "mla_decode_chunk",
    "mla_decode_chunk_workspace_bytes", "mla_decode_kernel_choice",
)
MLA_PAIRS_FULL, MLA_PAIRS_HIGH, MLA_PAIRS_UNIFORM, MLA_PAIRS_LOW = 0, 1, 2, 5
MLA_NOALLOC_SCRATCH_BYTES = 16 << 20


class MlaConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("r_pairs", ctypes.c_int32), ("d_c", ctypes.c_int32),
                ("rope_base", ctypes.c_double), ("softmax_scale", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("cache_kind", ctypes.c_int32)]


class MlaCache(ctypes.Structure):
    _fields_ = [("c_kv", ctypes.c_void_p), ("c_scales", ctypes.c_void_p),
                ("k_rope", ctypes.c_void_p), ("B", ctypes.c_int32), ("T_cap", ctypes.c_int32),
                ("c_resid", ctypes.c_void_p), ("resid_pos", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("n_blocks", ctypes.c_int32)]


class MlaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {_lib.mla_status_string(status).decode()} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with mha_mla_latent_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    cfgp, cachep = ctypes.POINTER(MlaConfig), ctypes.POINTER(MlaCache)
    sig = {
        "mla_status_string": (ctypes.c_char_p, [i32]),
        "mla_version": (ctypes.c_char_p, []),
        "mla_cache_bytes_per_token": (sz, [cfgp]),
        "mla_select_pairs": (i32, [cfgp, vp, vp, i32, vp, vp, vp]),
        "mla_fixed_pairs": (i32, [cfgp, i32, vp]),
        "mla_plan_create": (i32, [cfgp, vp, vp, vp, vp, vp, ctypes.POINTER(vp)]),
        "mla_plan_destroy": (None, [vp]),
        "mla_plan_set_option": (i32, [vp, i32, i64]),
        "mla_append": (i32, [vp, vp, vp, vp, i32, cachep, vp]),
        "mla_decode_workspace_bytes": (sz, [vp, i32]),
        "mla_decode_kernel_choice": (i32, [vp, cachep, ctypes.POINTER(i32)]),
        "mla_decode": (i32, [vp, cachep, vp, vp, i32, vp, vp, sz, vp]),
        "mla_device_error": (i32, [vp, ctypes.POINTER(i32)]),
        "mla_decode_noalloc": (i32, [vp, cachep, vp, vp, i32, vp, vp]),
        "mla_decode_step": (i32, [vp, cachep, vp, vp, vp, i32, vp, vp, sz, vp]),
        "mla_decode_chunk": (i32, [vp, cachep, vp, vp, i32, i32, vp, vp, sz, vp]),
        "mla_decode_chunk_workspace_bytes": (sz, [vp, i32, i32]),
        "mla_decode_step_host": (i32, [vp, cachep, vp, vp, vp, i32, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def _check(status, where):
    if status != MLA_OK:
        raise MlaError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensor must be contiguous")
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        if not t.flags["C_CONTIGUOUS"]:
            raise ValueError("array must be C-contiguous")
        return t.ctypes.data
    raise TypeError(type(t))


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def make_config(hidden, n_heads, n_kv_heads, head_dim, r_pairs, d_c, rope_base=10000.0,
                dtype="bf16", cache="same", resid=0, softmax_scale=0.0) -> MlaConfig:
    """cache: "same", "int4_g32" or "int2_g32"; resid: 0, or MLA_RESID_WINDOW for the int4
    cache with the unquantised residual window (MLA_CACHE_INT4_G32_R128); softmax_scale: 0
    for 1/sqrt(head_dim)."""
    if cache == "int2_g32":
        if resid:
            raise ValueError("the residual window is built for the int4 cache")
        kind = MLA_CACHE_INT2_G32
    elif cache == "int4_g32":
        if resid not in (0, MLA_RESID_WINDOW):
            raise ValueError(f"residual window {resid}: this library keeps {MLA_RESID_WINDOW} tokens")
        kind = MLA_CACHE_INT4_G32_R128 if resid else MLA_CACHE_INT4_G32
    else:
        if resid:
            raise ValueError("the residual window needs the int4 cache")
        kind = MLA_CACHE_SAME
    return MlaConfig(hidden, n_heads, n_kv_heads, head_dim, r_pairs, d_c, float(rope_base), float(softmax_scale),
                     MLA_BF16 if dtype == "bf16" else MLA_F32, kind)


def config_from_workload(wl) -> MlaConfig:
    return make_config(wl.hidden, wl.n_heads, wl.n_kv_heads, wl.head_dim, wl.r_pairs, wl.d_c,
                       wl.rope_base, wl.dtype, wl.cache, wl.resid)


def mla_version() -> str:
    return _lib.mla_version().decode()


def mla_status_string(status: int) -> str:
    return _lib.mla_status_string(status).decode()


def mla_cache_bytes_per_token(cfg: MlaConfig) -> int:
    return int(_lib.mla_cache_bytes_per_token(ctypes.byref(cfg)))


def mla_fixed_pairs(cfg: MlaConfig, strategy: int, check=True):
    """Fixed partial-RoPE pair set (MLA_PAIRS_*) -> numpy int32 [n_kv][r]."""
    out = np.zeros((cfg.n_kv_heads, max(cfg.r_pairs, 0)), dtype=np.int32)
    st = _lib.mla_fixed_pairs(ctypes.byref(cfg), int(strategy), out.ctypes.data_as(ctypes.c_void_p))
    if check:
        _check(st, "mla_fixed_pairs")
    return out if st == MLA_OK else None


def mla_select_pairs(cfg: MlaConfig, q_cal, k_cal, pair_idx, contrib=None, stream=None, check=True):
    st = _lib.mla_select_pairs(ctypes.byref(cfg), _ptr(q_cal), _ptr(k_cal), int(q_cal.shape[0]),
                               _ptr(pair_idx), _ptr(contrib), _stream(stream))
    if check:
        _check(st, "mla_select_pairs")
    return st


class Plan:
    """Owner of an mla_plan_t* (mla_plan_create / mla_plan_destroy)."""

    def __init__(self, handle, cfg):
        self.handle = handle
        self.cfg = cfg

    def __del__(self):
        self.close()

    def close(self):
        if getattr(self, "handle", None):
            if _lib is not None:   # module globals may already be gone at interpreter exit
                _lib.mla_plan_destroy(self.handle)
            self.handle = None


def mla_plan_create(cfg: MlaConfig, W_dkv, W_k, pair_idx, W_uk, W_uv) -> Plan:
    """Host arrays (torch CPU tensors or numpy) in the config dtype; pair_idx int32."""
    out = ctypes.c_void_p()
    keep = [W_dkv, W_k, pair_idx, W_uk, W_uv]  # noqa: F841  (alive during the call)
    st = _lib.mla_plan_create(ctypes.byref(cfg), _ptr(W_dkv), _ptr(W_k), _ptr(pair_idx),
                              _ptr(W_uk), _ptr(W_uv), ctypes.byref(out))
    _check(st, "mla_plan_create")
    return Plan(out.value, cfg)


def mla_plan_destroy(plan: Plan):
    plan.close()


def mla_plan_set_option(plan: Plan, option: int, value: int):
    _check(_lib.mla_plan_set_option(plan.handle, option, int(value)), "mla_plan_set_option")


def cache_struct(c_kv, c_scales, k_rope, B, T_cap, c_resid=None, resid_pos=None, block_table=None,
                 n_blocks=0) -> MlaCache:
    return MlaCache(_ptr(c_kv), _ptr(c_scales), _ptr(k_rope), int(B), int(T_cap), _ptr(c_resid),
                    _ptr(resid_pos), _ptr(block_table), int(n_blocks))


def mla_append(plan: Plan, x, seq_idx, pos, cache: MlaCache, stream=None, check=True):
    st = _lib.mla_append(plan.handle, _ptr(x), _ptr(seq_idx), _ptr(pos), int(x.shape[0]),
                         ctypes.byref(cache), _stream(stream))
    if check:
        _check(st, "mla_append")
    return st


def mla_decode_workspace_bytes(plan: Plan, B: int) -> int:
    return int(_lib.mla_decode_workspace_bytes(plan.handle, int(B)))


def mla_decode_kernel_choice(plan: Plan, cache: MlaCache) -> int:
    """The attention kernel mla_decode runs (1, 2 or 3, MLA_OPT_DECODE_KERNEL numbering)."""
    k = ctypes.c_int32(0)
    _check(_lib.mla_decode_kernel_choice(plan.handle, ctypes.byref(cache), ctypes.byref(k)), "mla_decode_kernel_choice")
    return int(k.value)


def mla_decode(plan: Plan, cache: MlaCache, seq_lens, q, out, workspace, stream=None, check=True):
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.mla_decode(plan.handle, ctypes.byref(cache), _ptr(seq_lens), _ptr(q), int(q.shape[0]),
                         _ptr(out), _ptr(workspace), ws_bytes, _stream(stream))
    if check:
        _check(st, "mla_decode")
    return st


def mla_decode_chunk_workspace_bytes(plan: Plan, B: int, Q: int) -> int:
    return int(_lib.mla_decode_chunk_workspace_bytes(plan.handle, int(B), int(Q)))


def mla_decode_chunk(plan: Plan, cache: MlaCache, seq_lens, q, out, workspace, stream=None, check=True):
    """Causal attention of each sequence's newest Q tokens: q and out are [B][Q][H][d_h]."""
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.mla_decode_chunk(plan.handle, ctypes.byref(cache), _ptr(seq_lens), _ptr(q), int(q.shape[0]),
                               int(q.shape[1]), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream))
    if check:
        _check(st, "mla_decode_chunk")
    return st


def mla_decode_step(plan: Plan, cache: MlaCache, seq_lens, x, q, out, workspace, stream=None, check=True):
    """Append every sequence's new token (row b of x at position seq_lens[b]-1 of sequence
    b) and decode every query, in one call (device tensors)."""
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.mla_decode_step(plan.handle, ctypes.byref(cache), _ptr(seq_lens), _ptr(x), _ptr(q), int(q.shape[0]),
                              _ptr(out), _ptr(workspace), ws_bytes, _stream(stream))
    if check:
        _check(st, "mla_decode_step")
    return st


def mla_decode_step_host(plan: Plan, cache: MlaCache, seq_lens, x, q, out, workspace, stream=None, check=True):
    """mla_decode_step with seq_lens, x, q and out in host memory (pinned torch CPU tensors
    or numpy arrays); the copies in and out are enqueued on the stream with the kernels."""
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.mla_decode_step_host(plan.handle, ctypes.byref(cache), _ptr(seq_lens), _ptr(x), _ptr(q),
                                   int(q.shape[0]), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream))
    if check:
        _check(st, "mla_decode_step_host")
    return st


def mla_decode_noalloc(plan: Plan, cache: MlaCache, seq_lens, q, out, stream=None, check=True):
    """mla_decode with the library's static scratch array as workspace (no allocation)."""
    st = _lib.mla_decode_noalloc(plan.handle, ctypes.byref(cache), _ptr(seq_lens), _ptr(q), int(q.shape[0]),
                                 _ptr(out), _stream(stream))
    if check:
        _check(st, "mla_decode_noalloc")
    return st


def mla_device_error(plan: Plan) -> int:
    code = ctypes.c_int32(0)
    _check(_lib.mla_device_error(plan.handle, ctypes.byref(code)), "mla_device_error")
    return int(code.value)
