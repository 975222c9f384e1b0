"""The fused decode step (mla_decode_step, mla_decode_step_host) against the oracle.

A step appends each sequence's newest token at position L_b - 1 and decodes its query
over [0, L_b).  The cache is prefilled with tokens [0, L_b - 1) by mla_append; the step
must then leave the same cache row at L_b - 1 as the oracle's append and the same output
as the oracle's decode (tolerances of the parity tests), through device buffers and
through host buffers.
"""

import numpy as np
import pytest
import torch

from tests.helpers import OracleCase, assert_close, assert_stored_close, plan_inputs, quant_scheme
from workloads import PARITY_WORKLOADS, generate as gen

pytestmark = pytest.mark.gpu

_CASES = {}


def case_for(wl):
    if wl.name not in _CASES:
        _CASES[wl.name] = OracleCase(wl)
    return _CASES[wl.name]


def prefilled(case, host_step):
    """Plan, cache holding tokens [0, L_b - 1) of every sequence, and the step's inputs."""
    import mha_mla_latent_b200 as mla
    from mha_mla_latent_b200.cache import LatentCache, workspace

    wl = case.wl
    cfg = mla.config_from_workload(wl)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    T_cap = int(max(case.lens))
    T_cap += T_cap % 2
    cache = LatentCache(cfg, wl.batch, T_cap, "cuda")
    for b in case.seqs:
        L = int(case.lens[b])
        if L > 1:
            x = case.tokens(b)[:L - 1]
            mla.mla_append(plan, gen.to_torch(x, wl.dtype, "cuda"),
                           torch.full((L - 1,), b, dtype=torch.int32, device="cuda"),
                           torch.arange(L - 1, dtype=torch.int32, device="cuda"), cache.struct)
    dev = "cpu" if host_step else "cuda"
    x = gen.to_torch(case.x_dec, wl.dtype, dev)
    q = gen.to_torch(case.q, wl.dtype, dev)
    lens = torch.tensor(case.lens, dtype=torch.int32, device=dev)
    out = torch.full_like(q, float("nan"))
    if host_step:
        x, q, lens, out = x.pin_memory(), q.pin_memory(), lens.pin_memory(), out.pin_memory()
    return mla, plan, cache, x, q, lens, out, workspace(plan, wl.batch)


STEP_WORKLOADS = [w for w in PARITY_WORKLOADS if int(np.min(gen.seq_lens(w))) >= 1]


@pytest.mark.parametrize("host_step", [False, True], ids=["device", "host"])
@pytest.mark.parametrize("wl", STEP_WORKLOADS, ids=[w.name for w in STEP_WORKLOADS])
def test_decode_step_matches_oracle(wl, host_step):
    case = case_for(wl)
    mla, plan, cache, x, q, lens, out, ws = prefilled(case, host_step)
    if host_step:
        mla.mla_decode_step_host(plan, cache.struct, lens, x, q, out, ws)
    else:
        mla.mla_decode_step(plan, cache.struct, lens, x, q, out, ws)
    torch.cuda.synchronize()
    assert mla.mla_device_error(plan) == 0
    got = out.double().cpu().numpy()
    for b in case.seqs:
        assert_close(got[b], case.reference(b), wl.dtype, f"{wl.name} step seq {b}")
        # the appended row at L-1
        p_ = int(case.lens[b]) - 1
        cc = case.cache[b]
        assert_stored_close(cache.k_rope_tokens(b, p_, p_ + 1)[0].double().cpu().numpy(), cc["kr_exact"][p_],
                            wl.dtype, f"kr {b}")
        qs = quant_scheme(wl)
        if qs is None:
            assert_stored_close(cache.latent_rows(b, p_, p_ + 1)[0].double().cpu().numpy(), cc["c_exact"][p_],
                                wl.dtype, f"c {b}")
        elif wl.resid:   # the new token owns its ring slot and the row holds its latent
            W = cache.resid_pos.shape[1]
            assert int(cache.resid_pos[b, p_ % W]) == p_
            assert_stored_close(cache.c_resid[b, p_ % W].double().cpu().numpy(), cc["c_exact"][p_],
                                wl.dtype, f"ring {b}")
    plan.close()


def test_decode_step_equals_append_then_decode():
    """Bit for bit: the fused step's output and cache equal mla_append + mla_decode."""
    wl = PARITY_WORKLOADS[2]
    case = case_for(wl)
    mla, plan, cache, x, q, lens, out, ws = prefilled(case, False)
    mla.mla_decode_step(plan, cache.struct, lens, x, q, out, ws)
    torch.cuda.synchronize()
    fused_c = cache.c_kv.clone()
    fused_kr = cache.k_rope.clone()
    _, plan2, cache2, _, _, _, out2, ws2 = prefilled(case, False)
    B = wl.batch
    mla.mla_append(plan2, x, torch.arange(B, dtype=torch.int32, device="cuda"), lens - 1, cache2.struct)
    mla.mla_decode(plan2, cache2.struct, lens, q, out2, ws2)
    torch.cuda.synchronize()
    assert torch.equal(fused_c, cache2.c_kv) and torch.equal(fused_kr, cache2.k_rope)
    assert torch.equal(out, out2)
    plan.close()
    plan2.close()
