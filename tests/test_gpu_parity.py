"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Tolerances: pair indices bit-exact; fp32 rel-L2 <= 1e-5; bf16/int4 decode outputs
rel-L2 <= 1e-2 and max-abs <= 3e-2.  Appended cache entries (stored in the config
dtype) are within one storage ulp of the exact value and rel-L2 <= 1e-2.  int4 codes
are bit-exact when the latent the kernel quantises is exact (one-hot tokens).
"""

import numpy as np
import pytest
import torch

import oracle as O
from tests.helpers import (OracleCase, assert_close, assert_stored_close, plan_inputs, quant_scheme,
                           upload_oracle_cache)
from workloads import PARITY_WORKLOADS, generate as gen

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mha_mla_latent_b200 as mla
    from mha_mla_latent_b200.cache import LatentCache, workspace

IDS = [w.name for w in PARITY_WORKLOADS]
_CASES = {}


def case_for(wl):
    if wl.name not in _CASES:
        _CASES[wl.name] = OracleCase(wl)
    return _CASES[wl.name]


def tc_kernel_ok(wl, kernel):
    """Kernel 2 (a token per softmax thread) takes bf16 with 32 heads; kernel 3 (a head per
    softmax thread) takes bf16 with up to 128 heads, GQA included, and up to 256 RoPE
    key columns."""
    if kernel == 2:
        return wl.dtype == "bf16" and wl.n_heads == 32
    if kernel == 3:
        return wl.dtype == "bf16" and wl.n_heads <= 128 and wl.n_kv_heads * 2 * wl.r_pairs <= 256
    return True


# 64 query heads: two per KV head (256 RoPE key columns), and eight per KV head over an int4 cache
WIDE_WORKLOADS = [PARITY_WORKLOADS[2].with_(name="h64_gqa2_dc128_small", n_heads=64, n_kv_heads=32, head_dim=64,
                                            d_c=128, fixed_lens=(900, 1, 200)),
                  PARITY_WORKLOADS[4].with_(name="h64_gqa8_int4_small", n_heads=64, n_kv_heads=8, head_dim=64,
                                            d_c=128, fixed_lens=(513, 64, 2))]


def make_plan(case, kernel=0, splits=0):
    cfg = mla.config_from_workload(case.wl)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    if kernel:
        mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_KERNEL, kernel)
    if splits:
        mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_SPLITS, splits)
    return cfg, plan


def run_decode(case, plan, cfg, cache=None, lens=None):
    wl = case.wl
    dev = "cuda"
    lens = case.lens if lens is None else lens
    T_cap = max(1, int(max(lens)))
    if cache is None:
        cache = LatentCache(cfg, wl.batch, T_cap, dev)
        upload_oracle_cache(case, cache, T_cap)
    seq = torch.tensor(np.asarray(lens), dtype=torch.int32, device=dev)
    q = gen.to_torch(case.q, wl.dtype, dev)
    out = torch.empty_like(q)
    ws = workspace(plan, wl.batch, dev)
    mla.mla_decode(plan, cache.struct, seq, q, out, ws)
    torch.cuda.synchronize()
    return out.double().cpu().numpy()


# --------------------------------------------------------------------------- a9
@pytest.mark.parametrize("wl", PARITY_WORKLOADS, ids=IDS)
def test_select_pairs_bit_exact(wl):
    case = case_for(wl)
    cfg = mla.config_from_workload(wl)
    q = gen.to_torch(case.q_cal, wl.dtype, "cuda")
    k = gen.to_torch(case.k_cal, wl.dtype, "cuda")
    from mha_mla_latent_b200.convert import select_pairs
    pair_idx, contrib = select_pairs(cfg, q, k)
    torch.cuda.synchronize()
    ref = case.conv["contrib"]
    # the seed must not be near-tied at the r-th/(r+1)-th boundary for a bit-exact claim
    srt = -np.sort(-ref, axis=1)
    gap = (srt[:, wl.r_pairs - 1] - srt[:, wl.r_pairs]) / srt[:, wl.r_pairs - 1]
    assert np.all(gap > 1e-4), f"near-tied seed: min relative gap {gap.min():.2e}"
    assert pair_idx.cpu().numpy().tolist() == case.conv["pair_idx"].tolist()
    np.testing.assert_allclose(contrib.cpu().numpy(), ref, rtol=2e-5)


# --------------------------------------------------------------------------- a0
@pytest.mark.parametrize("wl", PARITY_WORKLOADS, ids=IDS)
def test_append_parity(wl):
    case = case_for(wl)
    cfg, plan = make_plan(case)
    T_cap = int(max(case.lens))
    cache = LatentCache(cfg, wl.batch, max(T_cap, 1), "cuda")
    xs, sidx, pos = [], [], []
    for b in case.seqs:
        x = case.tokens(b)
        xs.append(x)
        sidx += [b] * x.shape[0]
        pos += list(range(x.shape[0]))
    x = gen.to_torch(np.concatenate(xs), wl.dtype, "cuda")
    mla.mla_append(plan, x, torch.tensor(sidx, dtype=torch.int32, device="cuda"),
                   torch.tensor(pos, dtype=torch.int32, device="cuda"), cache.struct)
    assert mla.mla_device_error(plan) == 0
    for b in case.seqs:
        L = int(case.lens[b])
        if L == 0:
            continue
        cc = case.cache[b]
        kr = cache.k_rope_tokens(b, 0, L).double().cpu().numpy()
        assert_stored_close(kr, cc["kr_exact"], wl.dtype, f"k_rope seq {b}")
        qs = quant_scheme(wl)
        if qs is not None:
            codes = qs[3](cache.latent_rows(b, 0, L).cpu().numpy())
            scales = cache.scale_rows(b, 0, L).cpu().numpy()
            deq = qs[1](codes, scales)
            assert_close(deq, qs[1](cc["codes"], cc["scales"]), wl.dtype, f"{wl.cache} latent seq {b}")
            # codes differ only where the float32 latents straddle a rounding boundary
            assert np.mean(codes != cc["codes"]) < 1e-3
            if wl.resid:
                _check_ring(cache, b, L, cc["c_exact"], wl)
        else:
            c = cache.latent_rows(b, 0, L).double().cpu().numpy()
            assert_stored_close(c, cc["c_exact"], wl.dtype, f"latent seq {b}")


@pytest.mark.parametrize("wl", PARITY_WORKLOADS, ids=IDS)
def test_append_decode_step_batch(wl):
    """The decode-step shape: one new token per sequence (N = B) appended at L_b - 1."""
    case = case_for(wl)
    cfg, plan = make_plan(case)
    T_cap = max(1, int(max(case.lens)))
    cache = LatentCache(cfg, wl.batch, T_cap, "cuda")
    seqs = [b for b in case.seqs if case.lens[b] > 0]
    x = np.stack([case.x_dec[b] for b in seqs])
    mla.mla_append(plan, gen.to_torch(x, wl.dtype, "cuda"), torch.tensor(seqs, dtype=torch.int32, device="cuda"),
                   torch.tensor([int(case.lens[b]) - 1 for b in seqs], dtype=torch.int32, device="cuda"),
                   cache.struct)
    assert mla.mla_device_error(plan) == 0
    for b in seqs:
        p_ = int(case.lens[b]) - 1
        cc = case.cache[b]
        assert_stored_close(cache.k_rope_tokens(b, p_, p_ + 1)[0].double().cpu().numpy(), cc["kr_exact"][p_],
                            wl.dtype, f"kr {b}")
        qs = quant_scheme(wl)
        if qs is not None:
            codes = qs[3](cache.latent_rows(b, p_, p_ + 1).cpu().numpy())
            deq = qs[1](codes, cache.scale_rows(b, p_, p_ + 1).cpu().numpy())
            assert_close(deq[0], qs[1](cc["codes"][p_:p_ + 1], cc["scales"][p_:p_ + 1])[0],
                         wl.dtype, f"{wl.cache} latent {b}")
            if wl.resid:   # only the appended token's slot is claimed and written
                W = cache.resid_pos.shape[1]
                tags = cache.resid_pos[b].cpu().numpy()
                assert tags[p_ % W] == p_ and np.sum(tags >= 0) == 1
                assert_stored_close(cache.c_resid[b, p_ % W].double().cpu().numpy(), cc["c_exact"][p_],
                                    wl.dtype, f"ring {b}")
        else:
            assert_stored_close(cache.latent_rows(b, p_, p_ + 1)[0].double().cpu().numpy(), cc["c_exact"][p_],
                                wl.dtype, f"c {b}")


def _check_ring(cache, b, L, c_exact, wl):
    """The ring after in-order appends of tokens [0, L): slot t % W holds token t for the
    W most recent tokens (tag t, row = the unquantised latent in the cache dtype); slots
    never written keep tag -1."""
    W = cache.resid_pos.shape[1]
    tags = cache.resid_pos[b].cpu().numpy()
    t = np.arange(max(0, L - W), L)
    np.testing.assert_array_equal(tags[t % W], t)
    if L < W:
        assert np.all(tags[L:] == -1)
    rows = cache.c_resid[b, t % W].double().cpu().numpy()
    assert_stored_close(rows, c_exact[t], wl.dtype, f"ring rows seq {b}")


RESID_WORKLOADS = [w for w in PARITY_WORKLOADS if w.resid]


@pytest.mark.parametrize("wl", RESID_WORKLOADS, ids=[w.name for w in RESID_WORKLOADS])
def test_residual_window_slides_with_decode_steps(wl):
    """Prefill in one call (positions wrap the ring several times: the newest token of
    each slot must win), then one-token decode steps; after each, the decode reads the
    128 most recent tokens unquantised and the rest as int4, as the oracle does."""
    case = case_for(wl)
    cfg, plan = make_plan(case)
    b = int(np.argmax(case.lens))
    x = case.tokens(b)
    L_end = x.shape[0]
    L0 = L_end - 80
    cache = LatentCache(cfg, 1, L_end, "cuda")
    mla.mla_append(plan, gen.to_torch(x[:L0], wl.dtype, "cuda"), torch.zeros(L0, dtype=torch.int32, device="cuda"),
                   torch.arange(L0, dtype=torch.int32, device="cuda"), cache.struct)
    cc = case.cache[b]
    _check_ring(cache, 0, L0, cc["c_exact"], wl)
    deq = O.dequant_int4_g32(cc["codes"], cc["scales"])
    plain = gen.cast(cc["c_exact"], wl.dtype)
    q = gen.to_torch(case.q[b:b + 1], wl.dtype, "cuda")
    out = torch.empty_like(q)
    ws = workspace(plan, 1, "cuda")
    checks = {L0 + 1, L_end - 59, L_end - 58, L_end}
    for L in range(L0 + 1, L_end + 1):
        mla.mla_append(plan, gen.to_torch(x[L - 1:L], wl.dtype, "cuda"), torch.zeros(1, dtype=torch.int32, device="cuda"),
                       torch.full((1,), L - 1, dtype=torch.int32, device="cuda"), cache.struct)
        if L not in checks:
            continue
        mla.mla_decode(plan, cache.struct, torch.tensor([L], dtype=torch.int32, device="cuda"), q, out, ws)
        torch.cuda.synchronize()
        c_mix = O.residual_window(deq[:L], plain[:L], wl.resid)
        ref = O.decode_unabsorbed(case.q[b], c_mix, cc["kr"][:L], case.conv["W_uk"], case.conv["W_uv"],
                                  case.conv["pair_idx"], case.theta)
        assert_close(out[0].double().cpu().numpy(), ref, wl.dtype, f"{wl.name} L={L}")
    assert mla.mla_device_error(plan) == 0
    _check_ring(cache, 0, L_end, cc["c_exact"], wl)


QUANT_WORKLOADS = [w for w in PARITY_WORKLOADS if w.cache != "same" and not w.resid]


@pytest.mark.parametrize("wl", QUANT_WORKLOADS, ids=[w.name for w in QUANT_WORKLOADS])
def test_append_quant_codes_bit_exact_on_exact_latents(wl):
    """One-hot tokens make c = a row of W_dkv exactly; codes and scales must match bit for bit."""
    case = case_for(wl)
    quant, _, pack, _ = quant_scheme(wl)
    cfg, plan = make_plan(case)
    n = 64
    x = np.zeros((n, wl.hidden))
    rows = np.arange(n) * 7 % wl.hidden
    x[np.arange(n), rows] = 1.0
    cache = LatentCache(cfg, 1, n, "cuda")
    mla.mla_append(plan, gen.to_torch(x, wl.dtype, "cuda"), torch.zeros(n, dtype=torch.int32, device="cuda"),
                   torch.arange(n, dtype=torch.int32, device="cuda"), cache.struct)
    torch.cuda.synchronize()
    c = case.conv["W_dkv"][rows]
    codes_ref, scales_ref = quant(c)
    np.testing.assert_array_equal(cache.c_kv[0].cpu().numpy(), pack(codes_ref))
    np.testing.assert_array_equal(cache.c_scales[0].cpu().numpy().view(np.uint16), scales_ref.view(np.uint16))


# --------------------------------------------------------------------------- a1-a8
@pytest.mark.parametrize("kernel", [0, 1, 2, 3])
@pytest.mark.parametrize("wl", PARITY_WORKLOADS, ids=IDS)
def test_decode_parity(wl, kernel):
    """kernel 0: the plan's choice; 1: CUDA-core split-K; 2: tcgen05, a token per softmax
    thread (bf16, 32 heads); 3: tcgen05, a head per softmax thread (bf16, up to 128 heads)."""
    case = case_for(wl)
    cfg, plan = make_plan(case, kernel=kernel)
    if not tc_kernel_ok(wl, kernel):
        with pytest.raises(mla.MlaError) as ei:
            run_decode(case, plan, cfg)
        assert ei.value.status == mla.MLA_ERR_UNSUPPORTED
        pytest.skip("outside this tensor-core kernel")
    got = run_decode(case, plan, cfg)
    assert mla.mla_device_error(plan) == 0
    for b in case.seqs:
        assert_close(got[b], case.reference(b), wl.dtype, f"decode seq {b} (L={case.lens[b]})")


@pytest.mark.parametrize("kernel", [0, 1, 3])
@pytest.mark.parametrize("wl", WIDE_WORKLOADS, ids=[w.name for w in WIDE_WORKLOADS])
def test_decode_parity_wide_heads(wl, kernel):
    """64 query heads: kernel 3 fills all 128 MMA rows with one query's heads."""
    case = case_for(wl)
    cfg, plan = make_plan(case, kernel=kernel)
    got = run_decode(case, plan, cfg)
    assert mla.mla_device_error(plan) == 0
    for b in case.seqs:
        assert_close(got[b], case.reference(b), wl.dtype, f"decode seq {b} (L={case.lens[b]})")


@pytest.mark.parametrize("kernel", [0, 3])
@pytest.mark.parametrize("wl", PARITY_WORKLOADS[2:4], ids=IDS[2:4])
def test_decode_split_invariance(wl, kernel):
    case = case_for(wl)
    outs = []
    for splits in (1, 2, 7, 0):
        cfg, plan = make_plan(case, kernel=kernel, splits=splits)
        outs.append(run_decode(case, plan, cfg))
    for o in outs[1:]:
        np.testing.assert_allclose(o, outs[0], rtol=0, atol=2e-2 if wl.dtype == "bf16" else 1e-6)


def test_decode_empty_and_overlong_sequences():
    wl = PARITY_WORKLOADS[2]
    case = case_for(wl)
    cfg, plan = make_plan(case)
    lens = np.array(case.lens)
    T_cap = int(lens.max())
    cache = LatentCache(cfg, wl.batch, T_cap, "cuda")
    upload_oracle_cache(case, cache, T_cap)
    bad = lens.copy()
    bad[1] = 0            # empty sequence -> zero row, no error
    got = run_decode(case, plan, cfg, cache=cache, lens=bad)
    assert mla.mla_device_error(plan) == 0
    assert np.all(got[1] == 0)
    assert_close(got[0], case.reference(0), wl.dtype, "seq 0 beside an empty sequence")
    bad[2] = T_cap + 5    # beyond capacity -> flagged, treated as empty
    got = run_decode(case, plan, cfg, cache=cache, lens=bad)
    assert mla.mla_device_error(plan) & mla.MLA_DEVERR_SEQ_LEN
    assert np.all(got[2] == 0)


# --------------------------------------------------------------------------- end to end
@pytest.mark.parametrize("wl", PARITY_WORKLOADS, ids=IDS)
def test_end_to_end_conversion_append_decode(wl):
    """Product conversion (GPU pair selection + device SVD) -> GPU append -> GPU decode,
    against the oracle's own conversion, append and decode from the same raw layer."""
    case = case_for(wl)
    from mha_mla_latent_b200.convert import convert_layer, plan_from_converted
    cfg = mla.config_from_workload(wl)
    conv = convert_layer(cfg, gen.to_torch(case.w["W_k"], wl.dtype, "cuda"),
                         gen.to_torch(case.w["W_v"], wl.dtype, "cuda"),
                         gen.to_torch(case.q_cal, wl.dtype, "cuda"), gen.to_torch(case.k_cal, wl.dtype, "cuda"))
    assert conv["pair_idx"].numpy().tolist() == case.conv["pair_idx"].tolist()
    plan = plan_from_converted(cfg, conv)
    T_cap = max(1, int(max(case.lens)))
    cache = LatentCache(cfg, wl.batch, T_cap, "cuda")
    for b in case.seqs:
        x = case.tokens(b)
        if x.shape[0] == 0:
            continue
        mla.mla_append(plan, gen.to_torch(x, wl.dtype, "cuda"),
                       torch.full((x.shape[0],), b, dtype=torch.int32, device="cuda"),
                       torch.arange(x.shape[0], dtype=torch.int32, device="cuda"), cache.struct)
    got = run_decode(case, plan, cfg, cache=cache)
    assert mla.mla_device_error(plan) == 0
    for b in case.seqs:
        assert_close(got[b], case.reference(b), wl.dtype, f"end-to-end seq {b}")


@pytest.mark.parametrize("wl,pairs", [(PARITY_WORKLOADS[2], "uniform"), (PARITY_WORKLOADS[2], "low"),
                                      (PARITY_WORKLOADS[1], "high"),
                                      (PARITY_WORKLOADS[0].with_(name="tiny_full_rope", r_pairs=16), "full")],
                         ids=["llama_uniform", "llama_low", "smollm_high", "tiny_full"])
def test_decode_parity_fixed_pair_sets(wl, pairs):
    """The other partial-RoPE strategies through the same conversion, plan and decode."""
    case = OracleCase(wl, pairs=pairs)
    cfg = mla.config_from_workload(wl)
    fixed = {"high": mla.MLA_PAIRS_HIGH, "low": mla.MLA_PAIRS_LOW, "uniform": mla.MLA_PAIRS_UNIFORM,
             "full": mla.MLA_PAIRS_FULL}[pairs]
    assert np.array_equal(mla.mla_fixed_pairs(cfg, fixed), case.conv["pair_idx"].astype(np.int32))
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    got = run_decode(case, plan, cfg)
    assert mla.mla_device_error(plan) == 0
    for b in case.seqs:
        assert_close(got[b], case.reference(b), wl.dtype, f"{pairs} decode seq {b}")


@pytest.mark.parametrize("wl", [PARITY_WORKLOADS[2], PARITY_WORKLOADS[1], PARITY_WORKLOADS[4]],
                         ids=["llama", "smollm", "int4"])
def test_svd_split_conversion_append_decode(wl):
    """SVD_split end to end: the product conversion (device SVDs) gives the oracle's pair set
    and decodes, after GPU append, to the oracle's SVD_split reference."""
    case = OracleCase(wl, svd="split")
    from mha_mla_latent_b200.convert import convert_layer, plan_from_converted
    cfg = mla.config_from_workload(wl)
    conv = convert_layer(cfg, gen.to_torch(case.w["W_k"], wl.dtype, "cuda"),
                         gen.to_torch(case.w["W_v"], wl.dtype, "cuda"),
                         gen.to_torch(case.q_cal, wl.dtype, "cuda"), gen.to_torch(case.k_cal, wl.dtype, "cuda"),
                         svd="split")
    assert conv["pair_idx"].numpy().tolist() == case.conv["pair_idx"].tolist()
    dk = wl.d_c // 2
    assert bool((conv["W_uk"][:, dk:] == 0).all()) and bool((conv["W_uv"][:, :dk] == 0).all())
    plan = plan_from_converted(cfg, conv)
    T_cap = max(1, int(max(case.lens)))
    cache = LatentCache(cfg, wl.batch, T_cap, "cuda")
    for b in case.seqs:
        x = case.tokens(b)
        if x.shape[0] == 0:
            continue
        mla.mla_append(plan, gen.to_torch(x, wl.dtype, "cuda"),
                       torch.full((x.shape[0],), b, dtype=torch.int32, device="cuda"),
                       torch.arange(x.shape[0], dtype=torch.int32, device="cuda"), cache.struct)
    got = run_decode(case, plan, cfg, cache=cache)
    assert mla.mla_device_error(plan) == 0
    for b in case.seqs:
        assert_close(got[b], case.reference(b), wl.dtype, f"SVD_split seq {b}")


# --------------------------------------------------------------------------- paged cache
def _paged_cache(cfg, B, lens, seed, spare=3):
    """A paged cache whose sequences' 128-token blocks sit at shuffled pool positions
    (plus spare blocks nobody uses); unused table entries name a spare block."""
    BT = mla.MLA_BLOCK_TOKENS
    T_cap = max(BT, -(-int(max(lens)) // BT) * BT)
    need = [-(-int(L) // BT) for L in lens]
    n_blocks = sum(need) + spare
    ids = np.random.default_rng(seed).permutation(n_blocks)
    table = np.full((B, T_cap // BT), ids[-1], dtype=np.int32)
    k = 0
    for b, nb in enumerate(need):
        table[b, :nb] = ids[k:k + nb]
        k += nb
    return LatentCache(cfg, B, T_cap, "cuda", block_table=table, n_blocks=n_blocks)


PAGED = [PARITY_WORKLOADS[0], PARITY_WORKLOADS[1], PARITY_WORKLOADS[2], PARITY_WORKLOADS[3],
         PARITY_WORKLOADS[4]] + RESID_WORKLOADS + [w for w in PARITY_WORKLOADS if w.cache == "int2_g32"]


@pytest.mark.parametrize("wl", PAGED, ids=[w.name for w in PAGED])
def test_paged_append_matches_contiguous(wl):
    """All tokens of all sequences in one append call, into a contiguous and a paged cache:
    every token's stored latent (or int4 codes and scales), RoPE keys and ring row agree
    bit for bit (the same arithmetic, only the addresses differ)."""
    case = case_for(wl)
    cfg, plan = make_plan(case)
    lens = [int(L) for L in case.lens]
    flat = LatentCache(cfg, wl.batch, max(1, max(lens)), "cuda")
    paged = _paged_cache(cfg, wl.batch, lens, seed=5)
    xs, sidx, pos = [], [], []
    for b in case.seqs:
        x = case.tokens(b)
        xs.append(x)
        sidx += [b] * x.shape[0]
        pos += list(range(x.shape[0]))
    x = gen.to_torch(np.concatenate(xs), wl.dtype, "cuda")
    si = torch.tensor(sidx, dtype=torch.int32, device="cuda")
    po = torch.tensor(pos, dtype=torch.int32, device="cuda")
    for c in (flat, paged):
        mla.mla_append(plan, x, si, po, c.struct)
    assert mla.mla_device_error(plan) == 0
    for b in case.seqs:
        L = lens[b]
        if L == 0:
            continue
        assert torch.equal(flat.latent_rows(b, 0, L), paged.latent_rows(b, 0, L)), f"latent seq {b}"
        if flat.c_scales is not None:
            assert torch.equal(flat.scale_rows(b, 0, L), paged.scale_rows(b, 0, L)), f"scales seq {b}"
        if flat.k_rope is not None:
            assert torch.equal(flat.k_rope_tokens(b, 0, L), paged.k_rope_tokens(b, 0, L)), f"k_rope seq {b}"
        if flat.c_resid is not None:
            assert torch.equal(flat.resid_pos[b], paged.resid_pos[b])
            assert torch.equal(flat.c_resid[b], paged.c_resid[b])


@pytest.mark.parametrize("kernel", [1, 2, 3])
@pytest.mark.parametrize("wl", PAGED, ids=[w.name for w in PAGED])
def test_paged_decode_parity(wl, kernel):
    """Decode over a paged cache (shuffled blocks) equals the decode over the contiguous
    cache bit for bit, and the oracle within tolerance."""
    if not tc_kernel_ok(wl, kernel):
        pytest.skip("outside this tensor-core kernel")
    case = case_for(wl)
    cfg, plan = make_plan(case, kernel=kernel)
    lens = [int(L) for L in case.lens]
    flat = run_decode(case, plan, cfg)
    paged = _paged_cache(cfg, wl.batch, lens, seed=7)
    upload_oracle_cache(case, paged, paged.T_cap)
    got = run_decode(case, plan, cfg, cache=paged)
    assert mla.mla_device_error(plan) == 0
    np.testing.assert_array_equal(got, flat)
    for b in case.seqs:
        assert_close(got[b], case.reference(b), wl.dtype, f"paged decode seq {b} (L={lens[b]})")


def test_paged_block_outside_pool_is_flagged():
    """A table entry outside the pool is reported (and block 0 read or written instead)."""
    wl = PARITY_WORKLOADS[2]
    case = case_for(wl)
    lens = [int(L) for L in case.lens]
    for kernel in (1, 2, 3):
        cfg, plan = make_plan(case, kernel=kernel)
        paged = _paged_cache(cfg, wl.batch, lens, seed=9)
        upload_oracle_cache(case, paged, paged.T_cap)
        paged.block_table[0, 0] = paged.n_blocks          # sequence 0's first block: outside
        run_decode(case, plan, cfg, cache=paged)
        assert mla.mla_device_error(plan) & mla.MLA_DEVERR_BLOCK
        x = gen.to_torch(case.x_dec[:1], wl.dtype, "cuda")
        mla.mla_append(plan, x, torch.zeros(1, dtype=torch.int32, device="cuda"),
                       torch.zeros(1, dtype=torch.int32, device="cuda"), paged.struct)
        assert mla.mla_device_error(plan) & mla.MLA_DEVERR_BLOCK


def test_cache_view_beyond_32bit_rows_is_refused():
    """A view of 2^31 token rows (B * T_cap, or n_blocks * 128 when paged) is refused before
    any launch.  The views describe small real arrays, and every access the calls would make
    (sequence 0, positions below 128, block 0) stays inside them."""
    wl = PARITY_WORKLOADS[2]
    case = case_for(wl)
    cfg, plan = make_plan(case)
    small = LatentCache(cfg, 2, 256, "cuda")
    table = torch.zeros(2, 2, dtype=torch.int32, device="cuda")
    views = [mla.cache_struct(small.c_kv, None, small.k_rope, 2, 1 << 30),
             mla.cache_struct(small.c_kv, None, small.k_rope, 2, 256, block_table=table, n_blocks=1 << 24)]
    x = gen.to_torch(case.x_dec[:1], wl.dtype, "cuda")
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    seq = torch.full((1,), 5, dtype=torch.int32, device="cuda")
    q = gen.to_torch(case.q[:1], wl.dtype, "cuda")
    out = torch.empty_like(q)
    ws = workspace(plan, 1, "cuda")
    for view in views:
        assert mla.mla_append(plan, x, zero, zero, view, check=False) == mla.MLA_ERR_UNSUPPORTED
        assert mla.mla_decode(plan, view, seq, q, out, ws, check=False) == mla.MLA_ERR_UNSUPPORTED
        assert mla.mla_decode_step(plan, view, seq, x, q, out, ws, check=False) == mla.MLA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert mla.mla_device_error(plan) == 0
    rows = mla.cache_struct(small.c_kv, None, small.k_rope, 2, 256)   # the real view still runs
    assert mla.mla_append(plan, x, zero, zero, rows, check=False) == mla.MLA_OK


# --------------------------------------------------------------------------- many queries per sequence
@pytest.mark.parametrize("wl,kernel", [(PARITY_WORKLOADS[2], 2), (PARITY_WORKLOADS[2], 1),
                                       (PARITY_WORKLOADS[1], 1), (PARITY_WORKLOADS[4], 2)],
                         ids=["llama_tc", "llama_cuda_core", "smollm_gqa", "int4_tc"])
def test_multi_query_causal_decode(wl, kernel):
    """A chunk of Q new tokens of one sequence attends causally in one call: query j, at
    position p_j, over tokens [0, p_j], through per-query rows of the block table that
    alias the sequence's blocks (the queries are the chunk tokens' own projections)."""
    case = case_for(wl)
    cfg, plan = make_plan(case, kernel=kernel)
    lens = [int(L) for L in case.lens]
    b = int(np.argmax(lens))
    L = lens[b]
    paged = _paged_cache(cfg, wl.batch, lens, seed=11)
    upload_oracle_cache(case, paged, paged.T_cap)
    Q = 12
    pos = np.arange(L - Q, L)
    x = case.tokens(b)
    q = gen.cast((x[pos] @ case.w["W_q"]).reshape(Q, wl.n_heads, wl.head_dim), wl.dtype)
    view = paged.query_view([b] * Q)
    out = torch.empty(Q, wl.n_heads, wl.head_dim, dtype=gen.torch_dtype(wl.dtype), device="cuda")
    mla.mla_decode(plan, view, torch.tensor(pos + 1, dtype=torch.int32, device="cuda"),
                   gen.to_torch(q, wl.dtype, "cuda"), out, workspace(plan, Q, "cuda"))
    torch.cuda.synchronize()
    assert mla.mla_device_error(plan) == 0
    got = out.double().cpu().numpy()
    cc = case.cache[b]
    for j, p in enumerate(pos):
        ref = O.decode_unabsorbed(q[j], cc["c"][:p + 1], cc["kr"][:p + 1], case.conv["W_uk"], case.conv["W_uv"],
                                  case.conv["pair_idx"], case.theta)
        assert_close(got[j], ref, wl.dtype, f"query at position {p}")


@pytest.mark.parametrize("kernel", [0, 1, 2])
@pytest.mark.parametrize("idx", [2, 4, 1], ids=["bf16_dc256", "int4_dc128", "gqa_smollm"])
def test_decode_softmax_scale(idx, kernel):
    """A config softmax_scale other than 1/sqrt(d_h) scales every score (every kernel that
    takes the shape: 0 the automatic choice, 1 CUDA cores, 2 token-row tcgen05)."""
    wl = PARITY_WORKLOADS[idx]
    if not tc_kernel_ok(wl, kernel):
        pytest.skip("outside this tensor-core kernel")
    case = case_for(wl)
    scale = 0.6 / np.sqrt(wl.head_dim)
    cfg = mla.make_config(wl.hidden, wl.n_heads, wl.n_kv_heads, wl.head_dim, wl.r_pairs, wl.d_c, wl.rope_base,
                          wl.dtype, wl.cache, wl.resid, softmax_scale=scale)
    plan = mla.mla_plan_create(cfg, **plan_inputs(case))
    if kernel:
        mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_KERNEL, kernel)
    got = run_decode(case, plan, cfg)
    assert mla.mla_device_error(plan) == 0
    for b in case.seqs:
        if case.lens[b] == 0:
            continue
        cc = case.cache[b]
        ref = O.decode_unabsorbed(case.q[b], cc["c"], cc["kr"], case.conv["W_uk"], case.conv["W_uv"],
                                  case.conv["pair_idx"], case.theta, scale=scale)
        assert_close(got[b], ref, wl.dtype, f"{wl.name} scale seq {b}")
        if case.lens[b] > 1:   # one token: its value whatever the scale
            assert not np.allclose(ref, case.reference(b), rtol=1e-3)
    plan.close()


def test_decode_kernel_choice():
    """The automatic choice runs the head-row tensor-core kernel wherever its shapes allow
    (bf16, up to 128 heads, GQA included), the CUDA-core kernel for fp32; forcing a kernel
    that cannot take the shape is reported."""
    for wl, want in ((PARITY_WORKLOADS[0], 1), (PARITY_WORKLOADS[1], 3), (PARITY_WORKLOADS[2], 3),
                     (PARITY_WORKLOADS[4], 3), (PARITY_WORKLOADS[6], 3), (PARITY_WORKLOADS[7], 3)):
        case = OracleCase(wl, seqs=[])
        cfg, plan = make_plan(case)
        cache = LatentCache(cfg, wl.batch, 256, "cuda")
        assert mla.mla_decode_kernel_choice(plan, cache.struct) == want, wl.name
        mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_KERNEL, 1)
        assert mla.mla_decode_kernel_choice(plan, cache.struct) == 1
        if wl.n_heads != 32 or wl.dtype == "f32":
            mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_KERNEL, 2)
            with pytest.raises(mla.MlaError) as ei:
                mla.mla_decode_kernel_choice(plan, cache.struct)
            assert ei.value.status == mla.MLA_ERR_UNSUPPORTED
        plan.close()
