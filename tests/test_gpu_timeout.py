"""The tensor-core kernel's bounded waits: a wait that runs out is reported, not hung on.

Every pipeline wait of the tensor-core decode kernel gives up after a bound
(MLA_OPT_WAIT_LIMIT_US).  The testing option MLA_OPT_TEST_SKIP_COPY leaves one latent
copy out in every CTA, so the waits for that tile run out: the call must come back,
flag MLA_DEVERR_TIMEOUT in the plan's error word (after draining its copies and
releasing its tensor memory), and the next decode on the same plan, with the option
cleared, must match the oracle again.  Nothing here faults or traps the GPU: the
missing copy is a barrier that nothing completes, and every wait on it is bounded.
"""

import numpy as np
import pytest
import torch

from tests.helpers import OracleCase, assert_close, plan_inputs, upload_oracle_cache
from workloads import PARITY_WORKLOADS, generate as gen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("idx,skip", [(2, 1), (2, 2), (4, 1)], ids=["bf16-first", "bf16-second", "int4-first"])
def test_wait_runs_out_then_plan_recovers(idx, skip):
    import mha_mla_latent_b200 as mla
    from mha_mla_latent_b200.cache import LatentCache, workspace

    # one sequence of 256 tokens: two tiles, each in its own CTA under the default split
    wl = PARITY_WORKLOADS[idx].with_(name=PARITY_WORKLOADS[idx].name + "_timeout", batch=1, fixed_lens=(256,))
    case = OracleCase(wl)
    cfg = mla.config_from_workload(wl)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_KERNEL, 2)
    if skip == 2:   # one worker for both tiles, so its second copy is the one left out
        mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_SPLITS, 1)
    T_cap = 256
    cache = LatentCache(cfg, 1, T_cap, "cuda")
    upload_oracle_cache(case, cache, T_cap)
    seq = torch.tensor(case.lens, dtype=torch.int32, device="cuda")
    q = gen.to_torch(case.q, wl.dtype, "cuda")
    out = torch.empty_like(q)
    ws = workspace(plan, 1)
    assert mla.mla_device_error(plan) == 0

    mla.mla_plan_set_option(plan, mla.MLA_OPT_WAIT_LIMIT_US, 2000)
    mla.mla_plan_set_option(plan, mla.MLA_OPT_TEST_SKIP_COPY, skip)
    mla.mla_decode(plan, cache.struct, seq, q, out, ws)
    err = mla.mla_device_error(plan)   # synchronises: the call came back
    assert err & mla.MLA_DEVERR_TIMEOUT, f"error word {err}: the wait did not run out"

    mla.mla_plan_set_option(plan, mla.MLA_OPT_TEST_SKIP_COPY, 0)
    mla.mla_plan_set_option(plan, mla.MLA_OPT_WAIT_LIMIT_US, 1_000_000)
    out.fill_(float("nan"))
    mla.mla_decode(plan, cache.struct, seq, q, out, ws)
    assert mla.mla_device_error(plan) == 0
    got = out.double().cpu().numpy()
    assert_close(got[0], case.reference(0), wl.dtype, f"{wl.name} after the timeout")
    plan.close()


def test_wait_limit_option_is_checked():
    import mha_mla_latent_b200 as mla

    wl = PARITY_WORKLOADS[2]
    case = OracleCase(wl, seqs=[])
    plan = mla.mla_plan_create(mla.config_from_workload(wl), **plan_inputs(case))
    for bad in (0, 99, 10_000_001):
        with pytest.raises(mla.MlaError):
            mla.mla_plan_set_option(plan, mla.MLA_OPT_WAIT_LIMIT_US, bad)
    with pytest.raises(mla.MlaError):
        mla.mla_plan_set_option(plan, mla.MLA_OPT_TEST_SKIP_COPY, -1)
    plan.close()
