"""Parity at the full workload sizes, in the launch configuration the bench times.

For each bf16 / int4 workload at its full size (batch, context lengths, hidden size),
the plan is built from the oracle's conversion, every sequence is prefilled through
mla_append, and one mla_decode runs over the whole batch with the kernel the plan picks
(the bench's configuration).  The oracle then decodes a few sampled sequences one by one
(float64) and their outputs are compared.  Only the sampled sequences need their exact
seeded context tokens: a sequence's output depends on its own cache rows alone, so the
other sequences are prefilled with device-random tokens through the same append path.
"""

import numpy as np
import pytest
import torch

import mha_mla_latent_b200 as mla
from mha_mla_latent_b200.cache import LatentCache, workspace
from tests.helpers import OracleCase, assert_close, plan_inputs
from workloads import generate as gen
from workloads import get

pytestmark = pytest.mark.gpu

FULL = ["smollm135m_gqa_bf16", "llama2_7b_bf16", "llama2_7b_ragged_bf16", "llama2_7b_int4", "llama2_7b_int4_r128",
        "llama2_7b_int2"]


def _sampled(wl, lens):
    b_long, b_short = int(np.argmax(lens)), int(np.argmin(lens))
    return sorted({0, wl.batch - 1, b_long, b_short})


@pytest.mark.parametrize("kernel", [0, 2], ids=["auto", "token_rows"])
@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_parity(name, kernel):
    """kernel 0: the plan's own choice (the head-row tcgen05 kernel on every workload here);
    2: the token-row tcgen05 kernel, on the workloads it takes (32 heads)."""
    wl = get(name)
    lens = gen.seq_lens(wl)
    T_cap = int(lens.max())
    T_cap += T_cap % 2
    cfg = mla.config_from_workload(wl)
    dev = "cuda"
    if kernel == 2 and wl.n_heads != 32:
        pytest.skip("the token-row tensor-core kernel takes 32 heads")
    seqs = _sampled(wl, lens)
    case = OracleCase(wl, seqs=seqs)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    if kernel:
        mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_KERNEL, kernel)
    cache = LatentCache(cfg, wl.batch, T_cap, dev)
    assert mla.mla_decode_kernel_choice(plan, cache.struct) == (kernel or 3)
    dt = gen.torch_dtype(wl.dtype)
    gpu_rng = torch.Generator(device=dev)
    gpu_rng.manual_seed(1234)
    chunk = 16384
    for b in range(wl.batch):
        L = int(lens[b])
        if L == 0:
            continue
        xb = case.tokens(b) if b in seqs else None
        for s in range(0, L, chunk):
            e = min(L, s + chunk)
            if xb is not None:
                xt = gen.to_torch(xb[s:e], wl.dtype, dev)
            else:
                xt = torch.randn(e - s, wl.hidden, generator=gpu_rng, device=dev).to(dt)
            mla.mla_append(plan, xt, torch.full((e - s,), b, dtype=torch.int32, device=dev),
                           torch.arange(s, e, dtype=torch.int32, device=dev), cache.struct)
    q = gen.to_torch(case.q, wl.dtype, dev)
    out = torch.empty_like(q)
    ws = workspace(plan, wl.batch, dev)
    mla.mla_decode(plan, cache.struct, torch.tensor(lens, dtype=torch.int32, device=dev), q, out, ws)
    torch.cuda.synchronize()
    assert mla.mla_device_error(plan) == 0
    got = out.double().cpu().numpy()
    for b in seqs:
        assert_close(got[b], case.reference(b), wl.dtype, f"{name} seq {b} (L={lens[b]})")
    plan.close()
