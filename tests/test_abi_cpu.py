"""C-ABI checks that need no GPU: the library loads, exports every declared entry point,
and rejects bad arguments with the documented status before touching the device."""

import ctypes

import numpy as np
import os
import re

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "mla_api.h")


@pytest.fixture(scope="module")
def mla():
    from mha_mla_latent_b200 import build
    build.build()
    import mha_mla_latent_b200._lib as lib
    return lib


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("mla_select_pairs", "mla_plan_create", "mla_append", "mla_decode",
              "mla_decode_workspace_bytes", "mla_device_error"):
        assert n in names


def test_every_entry_point_has_its_own_doc_comment():
    """Each MLA_API declaration sits right under a comment block that names it or documents
    it (argument meaning, layout, ownership, errors)."""
    lines = open(HEADER).read().splitlines()
    for i, line in enumerate(lines):
        m = re.match(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", line)
        if not m or line.startswith("#"):
            continue
        j = i - 1
        while j >= 0 and lines[j].strip() == "":
            j -= 1
        assert lines[j].rstrip().endswith("*/"), f"{m.group(1)}: no doc comment directly above"
        k = j
        while k >= 0 and not lines[k].lstrip().startswith("/*"):
            k -= 1
        block = " ".join(lines[k:j + 1])
        assert len(block) > 60, f"{m.group(1)}: doc comment too short"


def test_library_exports_every_declared_symbol(mla):
    so = ctypes.CDLL(mla.LIB_PATH)
    for name in declared_functions():
        assert hasattr(so, name), name
    assert set(declared_functions()) == set(mla.EXPORTED)


def test_status_strings_and_version(mla):
    assert "sm_100a" in mla.mla_version()
    for s in range(7):
        assert mla.mla_status_string(s)


def test_cache_bytes_per_token_matches_oracle_accounting(mla):
    import oracle as O
    from workloads import WORKLOADS
    for w in WORKLOADS:
        cfg = mla.config_from_workload(w)
        ref = O.cache_bytes_per_token(w.n_kv_heads, w.r_pairs, w.d_c, 4 if w.dtype == "f32" else 2,
                                      int4=w.cache == "int4_g32")
        assert mla.mla_cache_bytes_per_token(cfg) == ref, w.name


def test_invalid_configs_rejected(mla):
    ok = mla.make_config(512, 8, 4, 64, 4, 64)
    out = ctypes.c_void_p()
    bad = [
        mla.make_config(512, 9, 4, 64, 4, 64),       # H not a multiple of n_kv
        mla.make_config(512, 8, 4, 63, 4, 64),       # odd head dim
        mla.make_config(512, 8, 4, 64, 40, 64),      # r > d_h/2
        mla.make_config(0, 8, 4, 64, 4, 64),
    ]
    for cfg in bad:
        st = mla._lib.mla_plan_create(ctypes.byref(cfg), None, None, None, None, None, ctypes.byref(out))
        assert st == mla.MLA_ERR_INVALID_ARG
    f32_int4 = mla.make_config(512, 8, 4, 64, 4, 64, dtype="f32", cache="int4_g32")
    st = mla._lib.mla_plan_create(ctypes.byref(f32_int4), None, None, None, None, None, ctypes.byref(out))
    assert st == mla.MLA_ERR_UNSUPPORTED
    # null weights with a valid config
    st = mla._lib.mla_plan_create(ctypes.byref(ok), None, None, None, None, None, ctypes.byref(out))
    assert st == mla.MLA_ERR_INVALID_ARG
    assert mla._lib.mla_plan_create(ctypes.byref(ok), None, None, None, None, None, None) == mla.MLA_ERR_INVALID_ARG


def test_pair_selection_validation(mla):
    cfg = mla.make_config(512, 8, 4, 64, 4, 64)
    sp = mla._lib.mla_select_pairs
    assert sp(ctypes.byref(cfg), None, 4096, 16, 8192, None, None) == mla.MLA_ERR_INVALID_ARG
    assert sp(ctypes.byref(cfg), 4096, 4096, 0, 8192, None, None) == mla.MLA_ERR_INVALID_ARG
    assert sp(ctypes.byref(cfg), 4097, 4096, 16, 8192, None, None) == mla.MLA_ERR_ALIGNMENT


def test_append_and_decode_need_a_plan(mla):
    cache = mla.MlaCache(4096, None, 8192, 2, 16)
    assert mla._lib.mla_append(None, 4096, 4096, 4096, 1, ctypes.byref(cache), None) == mla.MLA_ERR_INVALID_ARG
    assert mla._lib.mla_decode(None, ctypes.byref(cache), 4096, 4096, 1, 4096, 4096, 1 << 20, None) \
        == mla.MLA_ERR_INVALID_ARG
    assert mla._lib.mla_decode_workspace_bytes(None, 4) == 0
    assert mla._lib.mla_plan_set_option(None, 1, 0) == mla.MLA_ERR_INVALID_ARG
    code = ctypes.c_int32()
    assert mla._lib.mla_device_error(None, ctypes.byref(code)) == mla.MLA_ERR_INVALID_ARG


@pytest.mark.parametrize("dh,r", [(32, 2), (64, 4), (128, 4), (128, 13)])
def test_fixed_pairs_match_oracle(mla, dh, r):
    """mla_fixed_pairs (library, host) equals the oracle's sets bit for bit."""
    import oracle as O
    cfg = mla.make_config(512, 8, 4, dh, r, 64)
    for name, code in (("high", mla.MLA_PAIRS_HIGH), ("low", mla.MLA_PAIRS_LOW),
                       ("uniform", mla.MLA_PAIRS_UNIFORM)):
        got = mla.mla_fixed_pairs(cfg, code)
        assert np.array_equal(got, O.fixed_pairs(name, dh, r, 4).astype(np.int32)), name
    full_cfg = mla.make_config(512, 8, 4, dh, dh // 2, 64)
    assert np.array_equal(mla.mla_fixed_pairs(full_cfg, mla.MLA_PAIRS_FULL),
                          O.fixed_pairs("full", dh, dh // 2, 4).astype(np.int32))
    assert mla.mla_fixed_pairs(cfg, mla.MLA_PAIRS_FULL, check=False) is None     # r != d_h / 2
    assert mla.mla_fixed_pairs(cfg, 3, check=False) is None                      # unknown strategy


def test_int2_and_residual_window_configs(mla):
    """2-bit cache accounting (d_c/4 code bytes + one fp16 scale per 32 + RoPE dims), the
    int2/int4 dtype rule, and the binding's cache-kind mapping."""
    import pytest
    c2 = mla.make_config(4096, 32, 32, 128, 4, 128, cache="int2_g32")
    assert c2.cache_kind == mla.MLA_CACHE_INT2_G32
    assert mla.mla_cache_bytes_per_token(c2) == 128 // 4 + 2 * (128 // 32) + 32 * 8 * 2
    c4r = mla.make_config(4096, 32, 32, 128, 4, 128, cache="int4_g32", resid=128)
    assert c4r.cache_kind == mla.MLA_CACHE_INT4_G32_R128
    assert mla.mla_cache_bytes_per_token(c4r) == 128 // 2 + 2 * (128 // 32) + 32 * 8 * 2
    out = ctypes.c_void_p()
    f32_int2 = mla.make_config(512, 8, 4, 64, 4, 64, dtype="f32", cache="int2_g32")
    st = mla._lib.mla_plan_create(ctypes.byref(f32_int2), None, None, None, None, None, ctypes.byref(out))
    assert st == mla.MLA_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        mla.make_config(512, 8, 4, 64, 4, 64, cache="int2_g32", resid=128)
    with pytest.raises(ValueError):
        mla.make_config(512, 8, 4, 64, 4, 64, cache="int4_g32", resid=64)


def test_cache_view_layout_matches_header(mla):
    """The ctypes mirror of mla_cache_t: field order and offsets of the C struct
    (three pointers, two int32, two pointers, a pointer and an int32)."""
    C = mla.MlaCache
    offs = {name: getattr(C, name).offset for name, _ in C._fields_}
    assert offs == {"c_kv": 0, "c_scales": 8, "k_rope": 16, "B": 24, "T_cap": 28, "c_resid": 32,
                    "resid_pos": 40, "block_table": 48, "n_blocks": 56}
    assert ctypes.sizeof(C) == 64


def test_binding_constants_match_the_header(mla):
    """Every enumerator and #define value of include/mla_api.h that the binding mirrors
    carries the same value on both sides (an ABI drift check)."""
    text = open(HEADER).read()
    body = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    values = {}
    for m in re.finditer(r"\b(MLA_[A-Z0-9_]+)\s*=\s*(\d+)", body):
        values[m.group(1)] = int(m.group(2))
    for m in re.finditer(r"#define\s+(MLA_[A-Z0-9_]+)\s+\(?(\d+)u?\s*(?:<<\s*(\d+))?\)?", body):
        v = int(m.group(2))
        values[m.group(1)] = v << int(m.group(3)) if m.group(3) else v
    mirrored = [n for n in values if hasattr(mla, n)]
    assert len(mirrored) >= 25, mirrored
    for n in mirrored:
        assert getattr(mla, n) == values[n], (n, getattr(mla, n), values[n])
    for n in ("MLA_CACHE_INT2_G32", "MLA_CACHE_INT4_G32_R128", "MLA_RESID_WINDOW", "MLA_BLOCK_TOKENS",
              "MLA_DEVERR_BLOCK", "MLA_NOALLOC_SCRATCH_BYTES"):
        assert n in mirrored, n


def test_cache_accessors_follow_the_documented_layout(mla):
    """LatentCache's token accessors (used by the parity tests to read and write the cache)
    against the layout mla_cache_t documents, on CPU tensors: contiguous rows [b][t], paged
    rows [block_table[b][t/128]][t%128], RoPE keys token-major at ((pb*cap + pt)*n_kv + g)*2r + j."""
    from mha_mla_latent_b200.cache import LatentCache
    import torch
    cfg = mla.make_config(256, 8, 4, 32, 2, 64, cache="int4_g32", resid=128)
    n_kv, r2, B = 4, 4, 3
    table = np.array([[5, 0, 2], [1, 4, 3], [6, 6, 6]], dtype=np.int32)
    caches = {"flat": LatentCache(cfg, B, 384, "cpu"),
              "paged": LatentCache(cfg, B, 384, "cpu", block_table=table, n_blocks=7)}
    rng = np.random.default_rng(1)
    for kind, c in caches.items():
        b, t0, n = 1, 100, 200                       # crosses the 128-token block boundary
        kr = torch.from_numpy(rng.standard_normal((n, n_kv, r2)).astype(np.float32))
        codes = torch.from_numpy(rng.integers(0, 256, size=(n, 32), dtype=np.uint8))
        c.set_k_rope_tokens(b, t0, kr)
        c.set_latent_rows(b, t0, codes)
        assert torch.equal(c.latent_rows(b, t0, t0 + n), codes)
        np.testing.assert_array_equal(c.k_rope_tokens(b, t0, t0 + n).float().numpy(),
                                      kr.to(torch.bfloat16).float().numpy())
        flat_kr = c.k_rope.reshape(-1).float().numpy()
        flat_c = c.c_kv.reshape(-1, 32).numpy()
        for i in (0, 27, 28, 150, 199):
            t = t0 + i
            if kind == "flat":
                pb, pt, cap = b, t, 384
            else:
                pb, pt, cap = int(table[b][t // 128]), t % 128, 128
            np.testing.assert_array_equal(flat_c[pb * cap + pt], codes[i].numpy())
            for g in range(n_kv):
                for j in range(r2):
                    off = ((pb * cap + pt) * n_kv + g) * r2 + j
                    assert flat_kr[off] == float(kr[i, g, j].to(torch.bfloat16))
    # per-query views alias a sequence's table row and keep the pool (no residual window:
    # its ring belongs to a sequence row)
    with pytest.raises(ValueError):
        caches["paged"].query_view([1])
    plain = LatentCache(mla.make_config(256, 8, 4, 32, 2, 64, cache="int4_g32"), B, 384, "cpu",
                        block_table=table, n_blocks=7)
    v = plain.query_view([1, 1, 0])
    assert v.B == 3 and v.n_blocks == 7 and v.T_cap == 384
    assert v._table_ref.tolist() == [table[1].tolist(), table[1].tolist(), table[0].tolist()]


def test_plain_c_host_program_links_and_runs(mla, tmp_path):
    """The boundary is a C ABI: a C99 program built with gcc -Wall -Werror against
    include/mla_api.h links the library and gets the documented results from the entry
    points that need no GPU."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = os.path.join(ROOT, "tests", "c_abi", "abi_host.c")
    exe = str(tmp_path / "abi_host")
    libdir = os.path.dirname(mla.LIB_PATH)
    name = os.path.basename(mla.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                    "-o", exe, "-L", libdir, f"-l:{name}", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "0 failed" in r.stdout
