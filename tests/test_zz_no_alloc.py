"""mla_decode_noalloc: the decode entry point for callers that cannot allocate device memory.

It runs the same kernels as mla_decode, with the workspace taken from a static array
inside the library instead of caller memory.  Checked through the C ABI against
mla_decode on the same inputs, on two calls in a row after a call with other inputs (the
array keeps the previous call's contents, so no call may depend on them).  This file is collected
last so a stop-at-first-failure run has already run every other test.
"""

import numpy as np
import pytest
import torch

from tests.helpers import OracleCase, assert_close, plan_inputs, upload_oracle_cache
from workloads import PARITY_WORKLOADS, generate as gen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("idx", [2, 4, 1], ids=["bf16_dc256", "int4_dc128", "gqa_smollm"])
def test_noalloc_decode_matches_decode_twice(idx):
    import mha_mla_latent_b200 as mla
    from mha_mla_latent_b200.cache import LatentCache, workspace

    wl = PARITY_WORKLOADS[idx]
    case = OracleCase(wl)
    cfg = mla.config_from_workload(wl)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    T_cap = int(max(case.lens))
    T_cap += T_cap % 2
    cache = LatentCache(cfg, wl.batch, T_cap, "cuda")
    upload_oracle_cache(case, cache, T_cap)
    seq = torch.tensor(case.lens, dtype=torch.int32, device="cuda")
    q = gen.to_torch(case.q, wl.dtype, "cuda")
    ref = torch.empty_like(q)
    ws = workspace(plan, wl.batch)
    assert mla.mla_decode_workspace_bytes(plan, wl.batch) <= mla.MLA_NOALLOC_SCRATCH_BYTES
    mla.mla_decode(plan, cache.struct, seq, q, ref, ws)
    torch.cuda.synchronize()
    ref_np = ref.double().cpu().numpy()
    # first fill the shared array with another call's contents: other queries and shorter
    # lengths give another split schedule, other partials and other absorbed queries, so
    # a read of anything the checked calls did not write themselves shows up as a mismatch
    other = torch.empty_like(q)
    mla.mla_decode_noalloc(plan, cache.struct, torch.clamp(seq // 2, min=1), -2.0 * q, other)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        mla.mla_decode_noalloc(plan, cache.struct, seq, q, out)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        for b in range(wl.batch):
            assert_close(got[b], ref_np[b], wl.dtype, f"no-alloc call {call} seq {b}")
    assert mla.mla_device_error(plan) == 0
    plan.close()


def test_noalloc_rejects_a_batch_beyond_the_scratch():
    import mha_mla_latent_b200 as mla
    from mha_mla_latent_b200.cache import LatentCache

    wl = PARITY_WORKLOADS[2]
    case = OracleCase(wl, seqs=[])
    cfg = mla.config_from_workload(wl)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    B = 4096  # needs far more than 16 MiB of partials
    assert mla.mla_decode_workspace_bytes(plan, B) > mla.MLA_NOALLOC_SCRATCH_BYTES
    cache = LatentCache(cfg, B, 2, "cuda")
    seq = torch.ones(B, dtype=torch.int32, device="cuda")
    q = torch.zeros(B, wl.n_heads, wl.head_dim, dtype=gen.torch_dtype(wl.dtype), device="cuda")
    out = torch.empty_like(q)
    st = mla.mla_decode_noalloc(plan, cache.struct, seq, q, out, check=False)
    assert st == mla.MLA_ERR_WORKSPACE_TOO_SMALL
    plan.close()


def test_noalloc_validates_the_cache_view_like_decode():
    """The same cache-view checks as mla_decode, before anything is launched: a paged view
    whose capacity is not a whole number of 128-token blocks, a block table without a pool
    size, and a residual-window field on a cache kind without a window are all refused."""
    import mha_mla_latent_b200 as mla
    from mha_mla_latent_b200 import _lib
    from mha_mla_latent_b200.cache import LatentCache

    wl = PARITY_WORKLOADS[2]
    case = OracleCase(wl, seqs=[])
    cfg = mla.config_from_workload(wl)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    cache = LatentCache(cfg, 2, 256, "cuda")
    table = torch.zeros(2, 2, dtype=torch.int32, device="cuda")
    seq = torch.ones(2, dtype=torch.int32, device="cuda")
    q = torch.zeros(2, wl.n_heads, wl.head_dim, dtype=gen.torch_dtype(wl.dtype), device="cuda")
    out = torch.empty_like(q)
    ring = torch.zeros(2, 128, wl.d_c, dtype=gen.torch_dtype(wl.dtype), device="cuda")
    bad = [
        _lib.cache_struct(cache.c_kv, None, cache.k_rope, 2, 200, block_table=table, n_blocks=4),
        _lib.cache_struct(cache.c_kv, None, cache.k_rope, 2, 256, block_table=table, n_blocks=0),
        _lib.cache_struct(cache.c_kv, None, cache.k_rope, 2, 256, c_resid=ring),
    ]
    for view in bad:
        assert mla.mla_decode_noalloc(plan, view, seq, q, out, check=False) == mla.MLA_ERR_INVALID_ARG
    plan.close()
