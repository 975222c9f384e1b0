"""Many queries per sequence (mla_decode_chunk) against the oracle, query by query.

Each sequence's newest Q tokens are its chunk: query i sits at position L - Q + i, is
rotated there and attends over tokens [0, L - Q + i].  The oracle decodes every query on
its own (float64, the unabsorbed definition) over its causal prefix; the chunk kernel's
outputs must match within the parity tolerances.  Chunk sizes cover a partial query block
(Q = 2), several blocks whose positions straddle 64-token tiles (Q = 12) and a long chunk
(Q = 64); lengths are not tile multiples; contiguous and paged caches; bf16, int4 and
2-bit latents; 32 heads (four queries per 128-row unit) and 9 GQA heads (fourteen).
"""

import os

import numpy as np
import pytest
import torch

import oracle as O
from tests.helpers import OracleCase, assert_close, plan_inputs, upload_oracle_cache
from workloads import PARITY_WORKLOADS, generate as gen

pytestmark = pytest.mark.gpu

WLS = [PARITY_WORKLOADS[2].with_(name="llama_dc256_chunk", fixed_lens=(1000, 333, 130)),
       PARITY_WORKLOADS[3].with_(name="llama_dc64_chunk", batch=3, fixed_lens=(2500, 129, 77)),
       PARITY_WORKLOADS[4].with_(name="llama_int4_chunk", fixed_lens=(700, 200, 77)),
       PARITY_WORKLOADS[7].with_(name="llama_int2_chunk", fixed_lens=(700, 130, 65)),
       PARITY_WORKLOADS[1].with_(name="smollm_gqa_chunk", fixed_lens=(300, 100, 70))]
_CASES = {}


def case_for(wl):
    if wl.name not in _CASES:
        _CASES[wl.name] = OracleCase(wl)
    return _CASES[wl.name]


def chunk_queries(case, Q):
    """q [B][Q][H][d_h]: the queries of each sequence's last Q tokens (the layer's own
    projection of those tokens, cast like every activation)."""
    wl = case.wl
    qs = []
    for b in case.seqs:
        x = case.tokens(b)[-Q:]
        qs.append(gen.project(x, case.w["W_q"], wl.dtype).reshape(Q, wl.n_heads, wl.head_dim))
    return np.stack(qs)


def reference(case, q, b, i, Q):
    L = int(case.lens[b])
    p = L - Q + i
    cc = case.cache[b]
    return O.decode_unabsorbed(q[b, i], cc["c"][:p + 1], cc["kr"][:p + 1], case.conv["W_uk"], case.conv["W_uv"],
                               case.conv["pair_idx"], case.theta)


def paged_cache(mla, cfg, B, lens, T_cap, seed):
    from mha_mla_latent_b200.cache import LatentCache
    BT = mla.MLA_BLOCK_TOKENS
    nb = T_cap // BT
    n_blocks = B * nb + 3
    perm = np.random.default_rng(seed).permutation(n_blocks)[:B * nb].reshape(B, nb).astype(np.int32)
    return LatentCache(cfg, B, T_cap, "cuda", block_table=perm, n_blocks=n_blocks)


@pytest.mark.parametrize("paged", [False, True], ids=["contiguous", "paged"])
@pytest.mark.parametrize("Q", [2, 12, 64])
@pytest.mark.parametrize("wl", WLS, ids=[w.name for w in WLS])
def test_chunk_matches_per_query_oracle(wl, Q, paged):
    import mha_mla_latent_b200 as mla
    from mha_mla_latent_b200.cache import LatentCache

    case = case_for(wl)
    cfg = mla.config_from_workload(wl)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    mla.mla_plan_set_option(plan, mla.MLA_OPT_WAIT_LIMIT_US, int(os.environ.get("MLA_TEST_WAIT_US", "1000000")))
    lens = [int(L) for L in case.lens]
    BT = mla.MLA_BLOCK_TOKENS
    T_cap = -(-max(lens) // BT) * BT
    cache = paged_cache(mla, cfg, wl.batch, lens, T_cap, 11) if paged else LatentCache(cfg, wl.batch, T_cap, "cuda")
    upload_oracle_cache(case, cache, T_cap)
    q = chunk_queries(case, Q)
    qt = gen.to_torch(q, wl.dtype, "cuda")
    out = torch.full_like(qt, float("nan"))
    ws = torch.empty(mla.mla_decode_chunk_workspace_bytes(plan, wl.batch, Q), dtype=torch.uint8, device="cuda")
    mla.mla_decode_chunk(plan, cache.struct, torch.tensor(lens, dtype=torch.int32, device="cuda"), qt, out, ws)
    torch.cuda.synchronize()
    err = mla.mla_device_error(plan)
    assert err == 0, f"device error word {err}"
    got = out.double().cpu().numpy()
    for b in case.seqs:
        for i in sorted({0, 1, Q // 2, Q - 2, Q - 1}):
            assert_close(got[b, i], reference(case, q, b, i, Q), wl.dtype, f"{wl.name} Q={Q} seq {b} query {i}")
    plan.close()


def test_chunk_of_one_is_decode():
    """Q = 1 is the decode itself."""
    import mha_mla_latent_b200 as mla
    from mha_mla_latent_b200.cache import LatentCache, workspace

    wl = WLS[0]
    case = case_for(wl)
    cfg = mla.config_from_workload(wl)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    T_cap = int(max(case.lens))
    cache = LatentCache(cfg, wl.batch, T_cap, "cuda")
    upload_oracle_cache(case, cache, T_cap)
    seq = torch.tensor(case.lens, dtype=torch.int32, device="cuda")
    q = gen.to_torch(case.q, wl.dtype, "cuda")
    ref, out = torch.empty_like(q), torch.empty_like(q)
    ws = workspace(plan, wl.batch)
    mla.mla_decode(plan, cache.struct, seq, q, ref, ws)
    mla.mla_decode_chunk(plan, cache.struct, seq, q.unsqueeze(1), out.unsqueeze(1), ws)
    torch.cuda.synchronize()
    assert torch.equal(ref, out)
    plan.close()


def test_chunk_rejects_bad_arguments():
    import mha_mla_latent_b200 as mla
    from mha_mla_latent_b200.cache import LatentCache

    wl = WLS[0]
    case = OracleCase(wl, seqs=[])
    cfg = mla.config_from_workload(wl)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    cache = LatentCache(cfg, 2, 256, "cuda")
    seq = torch.full((2,), 100, dtype=torch.int32, device="cuda")
    q = torch.zeros(2, 300, wl.n_heads, wl.head_dim, dtype=torch.bfloat16, device="cuda")   # Q > T_cap
    out = torch.empty_like(q)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    assert mla.mla_decode_chunk(plan, cache.struct, seq, q, out, ws, check=False) == mla.MLA_ERR_INVALID_ARG
    q = q[:, :8].contiguous()
    out = torch.empty_like(q)
    assert mla.mla_decode_chunk(plan, cache.struct, seq, q, out, ws[:16], check=False) == \
        mla.MLA_ERR_WORKSPACE_TOO_SMALL
    plan.close()
