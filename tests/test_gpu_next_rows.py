"""GPU parity of the rows next to the decode path, through the C ABI, against
the fp64 oracle, element by element:

- W_UV absorbed into the output projection: W_OV = W_O blockdiag(W_UV_h)
  (DeepSeek-V2 explainer, section 3 remark; MLA walk-through, section 1 step 5)
  and y = W_OV o_lat;
- merged-matrix absorption W_UQK_h = W_UK_h^T W_UQ_h (walk-through, section 3
  order B) and the query chain that uses it;
- the fused front end (append and absorb from one read of h; walk-through,
  section 1 steps 1 and 3): exactly the predicted cache slots change;
- the failure-path self-test: a kernel whose bounded wait runs out reports
  MLA_ERR_TIMEOUT and leaves the context usable.
"""
import numpy as np
import pytest

from mla_latent_kv_33_b200 import synth

pytestmark = pytest.mark.gpu

V2 = synth.WORKLOADS["v2_b64_paged"]
V3 = synth.WORKLOADS["v3_b128_nq2"]
TINY = synth.WORKLOADS["tiny_fp32"]
TINY_BF16 = synth.shrink(TINY, dtype="bf16")
V2_SMALL_D = synth.shrink(V2, d=512)  # tensor-core geometry with a narrow model width


@pytest.fixture(scope="module")
def mla():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mla_latent_kv_33_b200 import mla as m
    return m


def _stored(rng_vals, dtype):
    """(float64 values exactly representable in storage, device tensor)."""
    from tests.gpu_util import dev
    vals, bits = synth._round_store(np.asarray(rng_vals, np.float32), dtype)
    return vals.astype(np.float64), dev(bits if dtype == "bf16" else vals, dtype)


def _tdt(torch, w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


# ------------------------------------------------- W_UV absorbed into W_O ----

@pytest.mark.parametrize("w", [V2_SMALL_D, TINY, TINY_BF16], ids=["v2_d512", "tiny_fp32", "tiny_bf16"])
def test_absorb_wo_and_latent_o_proj_match_oracle(mla, orc, w):
    import torch
    from tests.gpu_util import assert_close, dims_of, host, orc_dims_of
    p, po = dims_of(w, mla), orc_dims_of(w, orc)
    HD, HC = w.n_h * w.d_h, w.n_h * w.d_c
    rng = np.random.default_rng(31)
    W_O, W_O_d = _stored(rng.standard_normal((w.d, HD)), w.dtype)  # unit entries: W_OV is O(1)
    W_UV, W_UV_d = _stored(rng.standard_normal((HD, w.d_c)) / np.sqrt(w.d_c), w.dtype)
    W_OV_d = torch.full((w.d, HC), float("nan"), device="cuda", dtype=_tdt(torch, w))
    mla.mla_absorb_wo(p, W_O_d, W_UV_d, W_OV_d)
    assert mla.mla_get_device_error() == mla.MLA_OK
    W_OV = orc.absorb_wo(po, W_O, W_UV)
    assert_close(host(W_OV_d), W_OV, "W_OV")
    # W_OV is a stored weight: the oracle's own chain rounds it once to the storage format
    W_OV_stored = synth.bf16_to_f32(synth.bf16_bits(W_OV.astype(np.float32))) if w.dtype == "bf16" else W_OV
    for T in (5, 200):
        o_lat, o_lat_d = _stored(rng.standard_normal((T, w.n_h, w.d_c)) * 0.05, w.dtype)
        y = torch.full((T, w.d), float("nan"), device="cuda", dtype=_tdt(torch, w))
        mla.mla_o_proj_latent(p, o_lat_d, W_OV_d, y)
        assert mla.mla_get_device_error() == mla.MLA_OK
        # this op on the GPU's own W_OV, and the oracle's whole chain (its W_OV, stored)
        assert_close(host(y), orc.o_proj(host(W_OV_d), o_lat.reshape(T, HC)), f"y = W_OV o_lat (T={T})")
        assert_close(host(y), orc.o_proj(W_OV_stored, o_lat.reshape(T, HC)), f"y, oracle chain (T={T})")


def test_absorb_wo_full_width_sampled_rows(mla, orc):
    import torch
    from tests.gpu_util import assert_close, dims_of, host, orc_dims_of
    w = V2
    p = dims_of(w, mla)
    HD, HC = w.n_h * w.d_h, w.n_h * w.d_c
    rng = np.random.default_rng(32)
    W_O, W_O_d = _stored(rng.standard_normal((w.d, HD)), w.dtype)
    W_UV, W_UV_d = _stored(rng.standard_normal((HD, w.d_c)) / np.sqrt(w.d_c), w.dtype)
    W_OV_d = torch.empty((w.d, HC), device="cuda", dtype=torch.bfloat16)
    mla.mla_absorb_wo(p, W_O_d, W_UV_d, W_OV_d)
    assert mla.mla_get_device_error() == mla.MLA_OK
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, w.d - 1], rng.integers(0, w.d, 40)]))
    po = orc_dims_of(synth.shrink(w, d=len(rows)), orc)
    assert_close(host(W_OV_d[torch.from_numpy(rows).cuda()]), orc.absorb_wo(po, W_O[rows], W_UV),
                 "W_OV (sampled rows)")


# ------------------------------------------------- merged-matrix absorption ----

@pytest.mark.parametrize("w", [V2, TINY], ids=["v2", "tiny_fp32"])
def test_absorb_merge_matches_oracle(mla, orc, w):
    import torch
    from tests.gpu_util import assert_close, dims_of, host, orc_dims_of
    p, po = dims_of(w, mla), orc_dims_of(w, orc)
    HD = w.n_h * w.d_h
    rng = np.random.default_rng(33)
    W_UQ, W_UQ_d = _stored(rng.standard_normal((HD, w.d_cq)), w.dtype)  # unit entries: W_UQK is O(10)
    W_UK, W_UK_d = _stored(rng.standard_normal((HD, w.d_c)), w.dtype)
    W_UQK_d = torch.full((w.n_h * w.d_c, w.d_cq), float("nan"), device="cuda", dtype=_tdt(torch, w))
    mla.mla_absorb_merge(p, W_UQ_d, W_UK_d, W_UQK_d)
    assert mla.mla_get_device_error() == mla.MLA_OK
    assert_close(host(W_UQK_d), orc.absorb_merge(po, W_UQ, W_UK), "W_UQK")


MERGED_CASES = {
    "v2_T5": synth.shrink(V2, B=5, L_lo=1, L_hi=300),
    "v2_T200": synth.shrink(V2, B=200, L_lo=1, L_hi=100),
    "v3_T256_nq2": synth.shrink(V3, L_lo=2, L_hi=150, median=60.0),
    "tiny_fp32": TINY,
}


@pytest.mark.parametrize("case", list(MERGED_CASES))
def test_absorb_q_merged_matches_two_stage_oracle(mla, orc, case):
    import torch
    from tests.gpu_util import assert_close, dims_of, host, orc_dims_of, store
    w = MERGED_CASES[case]
    x = synth.generate(w, seed=104)
    p = dims_of(w, mla)
    W = {k: store(x.weights[k], x.weights_bits.get(k), w.dtype) for k in ("W_DQ", "W_UQ", "W_QR", "W_UK")}
    W_UQK = torch.empty((w.n_h * w.d_c, w.d_cq), device="cuda", dtype=_tdt(torch, w))
    mla.mla_absorb_merge(p, W["W_UQ"], W["W_UK"], W_UQK)
    q = torch.full((w.T, w.n_h, w.D), float("nan"), device="cuda", dtype=_tdt(torch, w))
    mla.mla_absorb_q_merged(p, store(x.h, x.h_bits, w.dtype), W["W_DQ"], W_UQK, W["W_QR"],
                            torch.from_numpy(x.positions).cuda(), q)
    assert mla.mla_get_device_error() == mla.MLA_OK
    ref = orc.absorb_q(orc_dims_of(w, orc), x.h, x.weights["W_DQ"], x.weights["W_UQ"], x.weights["W_QR"],
                       x.weights["W_UK"], x.positions)
    assert_close(host(q), ref, "q (merged absorption) vs the two-stage oracle")


# ------------------------------------------------------ fused front end ----

FRONT_CASES = {
    "v2_paged_T5": synth.shrink(V2, B=5, L_lo=1, L_hi=300),
    "v2_paged_T64": synth.shrink(V2, B=64, L_lo=1, L_hi=200),
    "v3_paged_T6_nq2": synth.shrink(V3, B=3, L_lo=2, L_hi=200),
    "v3_paged_T256_nq2": synth.shrink(V3, L_lo=2, L_hi=150, median=60.0),
    "v2_contig_T3": synth.shrink(synth.WORKLOADS["v2_b16_4k"], B=3, L=77),
    "tiny_fp32": TINY,
}


@pytest.mark.parametrize("case", list(FRONT_CASES))
def test_front_end_matches_oracle_and_writes_exact_slots(mla, orc, case):
    import torch
    from tests.gpu_util import assert_close, cache_host, dev, dims_of, host, orc_dims_of, store
    w = FRONT_CASES[case]
    x = synth.generate(w, seed=105)
    p = dims_of(w, mla)
    W = {k: store(x.weights[k], x.weights_bits.get(k), w.dtype) for k in x.weights}
    cache_t = dev(x.cache, w.dtype)
    before = x.cache.copy()
    bt = None if x.block_table is None else torch.from_numpy(x.block_table).cuda()
    cache = mla.Cache(cache_t, bt)
    q = torch.full((w.T, w.n_h, w.D), float("nan"), device="cuda", dtype=_tdt(torch, w))
    pos = torch.from_numpy(x.positions).cuda()
    mla.mla_front_end(p, store(x.h, x.h_bits, w.dtype), W["W_DKV"], W["W_KR"], W["W_DQ"], W["W_UQ"], W["W_QR"],
                      W["W_UK"], torch.from_numpy(x.seq_idx).cuda(), pos, cache, q)
    assert mla.mla_get_device_error() == mla.MLA_OK
    po = orc_dims_of(w, orc)
    after = cache_host(cache_t, w.dtype)
    oc = orc.Cache(before, x.block_table)
    slots = [oc.slot(int(x.seq_idx[t]), int(x.positions[t])) for t in range(w.T)]
    view = np.uint16 if w.dtype == "bf16" else np.uint32
    flat_b, flat_a = before.reshape(-1, w.D), after.reshape(-1, w.D)
    changed = np.nonzero(np.any(flat_a.view(view) != flat_b.view(view), axis=1))[0]
    assert sorted(changed.tolist()) == sorted(slots), "the front end touched rows other than the predicted slots"
    got = flat_a[slots]
    got = synth.bf16_to_f32(got) if w.dtype == "bf16" else got
    assert_close(got, orc.append_rows(po, x.h, x.weights["W_DKV"], x.weights["W_KR"], x.positions), "appended rows")
    ref_q = orc.absorb_q(po, x.h, x.weights["W_DQ"], x.weights["W_UQ"], x.weights["W_QR"], x.weights["W_UK"],
                         x.positions)
    assert_close(host(q), ref_q, "q")


# ------------------------------------------------ failure-path self-test ----

def test_timed_out_wait_is_reported_and_the_context_stays_usable(mla, orc):
    import torch
    from tests.gpu_util import assert_close, dev, dims_of, host, orc_dims_of, store
    scratch = torch.zeros(65536, dtype=torch.uint8, device="cuda")
    assert mla.mla_get_device_error() == mla.MLA_OK
    mla.mla_selftest_timeout(2000, scratch)  # 2 us: the kernel's first wait runs out
    assert mla.mla_get_device_error() == mla.MLA_ERR_TIMEOUT
    assert mla.mla_get_device_error() == mla.MLA_OK  # the word is cleared on read
    # a normal call afterwards still computes the right result
    w = synth.shrink(V2, B=3, L_lo=1, L_hi=50)
    x = synth.generate(w, seed=106)
    rng = np.random.default_rng(8)
    vals, bits = synth._round_store(rng.standard_normal((w.T, w.n_h, w.d_c)).astype(np.float32) * 0.05, w.dtype)
    o = torch.empty((w.T, w.n_h * w.d_h), device="cuda", dtype=torch.bfloat16)
    mla.mla_out_proj(dims_of(w, mla), dev(bits, w.dtype), store(x.weights["W_UV"], x.weights_bits["W_UV"], w.dtype), o)
    assert mla.mla_get_device_error() == mla.MLA_OK
    assert_close(host(o), orc.out_proj(orc_dims_of(w, orc), vals, x.weights["W_UV"]), "o after the self-test")
