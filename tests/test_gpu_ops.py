"""GPU parity of mla_cache_append, mla_absorb_q and mla_out_proj against the
fp64 oracle. Cache indexing is checked bit-exactly: exactly the predicted
slots change, every other byte keeps its canary."""
import numpy as np
import pytest

from mla_latent_kv_33_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mla():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mla_latent_kv_33_b200 import mla as m
    return m


def _weights(x, dt):
    from tests.gpu_util import store
    return {k: store(x.weights[k], x.weights_bits.get(k), dt) for k in x.weights}


CASES = {
    "v2_paged_T5": synth.shrink(synth.WORKLOADS["v2_b64_paged"], B=5, L_lo=1, L_hi=300),
    "v3_paged_T6_nq2": synth.shrink(synth.WORKLOADS["v3_b128_nq2"], B=3, L_lo=2, L_hi=200),
    "v2_contig_T3": synth.shrink(synth.WORKLOADS["v2_b16_4k"], B=3, L=77),
    # 256 token rows: the absorb runs as [W_UQ; W_QR] then the per-head W_UK^T GEMM through the workspace
    "v3_paged_T256_nq2": synth.shrink(synth.WORKLOADS["v3_b128_nq2"], L_lo=2, L_hi=150, median=60.0),
    "tiny_fp32": synth.WORKLOADS["tiny_fp32"],
    "small_bf16": synth.Workload("small_bf16", 9, d=96, n_h=3, d_h=16, d_c=32, d_cq=48, d_r=8, B=4,
                                 n_q=1, lens="uniform", L_lo=1, L_hi=40, paged=True, block_size=16),
}


@pytest.mark.parametrize("case", list(CASES))
def test_append_writes_exact_slots(mla, orc, case):
    import torch
    from tests.gpu_util import assert_close, cache_host, dev, dims_of, orc_dims_of, store
    w = CASES[case]
    x = synth.generate(w, seed=100)
    if w.prefill == "append":   # canary-only cache for this test
        pass
    W = _weights(x, w.dtype)
    h = store(x.h, x.h_bits, w.dtype)
    cache_t = dev(x.cache, w.dtype)
    before = x.cache.copy()
    bt = None if x.block_table is None else torch.from_numpy(x.block_table).cuda()
    cache = mla.Cache(cache_t, bt)
    p = dims_of(w, mla)
    mla.mla_cache_append(p, h, W["W_DKV"], W["W_KR"], torch.from_numpy(x.seq_idx).cuda(),
                         torch.from_numpy(x.positions).cuda(), cache)
    assert mla.mla_get_device_error() == mla.MLA_OK
    after = cache_host(cache_t, w.dtype)
    po = orc_dims_of(w, orc)
    oc = orc.Cache(before, x.block_table)
    rows_ref = orc.append_rows(po, x.h, x.weights["W_DKV"], x.weights["W_KR"], x.positions)
    flat_b = before.reshape(-1, w.D)
    flat_a = after.reshape(-1, w.D)
    slots = [oc.slot(int(x.seq_idx[t]), int(x.positions[t])) for t in range(w.T)]
    assert len(set(slots)) == len(slots)
    changed = np.nonzero(np.any(flat_a.view(np.uint16 if w.dtype == "bf16" else np.uint32) !=
                                flat_b.view(np.uint16 if w.dtype == "bf16" else np.uint32), axis=1))[0]
    assert sorted(changed.tolist()) == sorted(slots), "append touched rows other than the predicted slots"
    got = flat_a[slots]
    got = synth.bf16_to_f32(got) if w.dtype == "bf16" else got
    assert_close(got, rows_ref, "appended rows")


@pytest.mark.parametrize("case", list(CASES))
def test_absorb_matches_oracle(mla, orc, case):
    import torch
    from tests.gpu_util import assert_close, dims_of, host, orc_dims_of, store
    w = CASES[case]
    x = synth.generate(w, seed=101)
    W = _weights(x, w.dtype)
    h = store(x.h, x.h_bits, w.dtype)
    q = torch.full((w.T, w.n_h, w.D), float("nan"), device="cuda",
                   dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32)
    p = dims_of(w, mla)
    mla.mla_absorb_q(p, h, W["W_DQ"], W["W_UQ"], W["W_QR"], W["W_UK"], torch.from_numpy(x.positions).cuda(), q)
    assert mla.mla_get_device_error() == mla.MLA_OK
    ref = orc.absorb_q(orc_dims_of(w, orc), x.h, x.weights["W_DQ"], x.weights["W_UQ"], x.weights["W_QR"],
                       x.weights["W_UK"], x.positions)
    assert_close(host(q), ref, "q = [q_lat | q_R]")


@pytest.mark.parametrize("case", list(CASES))
def test_out_proj_matches_oracle(mla, orc, case):
    import torch
    from tests.gpu_util import assert_close, dev, dims_of, host, orc_dims_of, store
    w = CASES[case]
    x = synth.generate(w, seed=102)
    rng = np.random.default_rng(7)
    vals, bits = synth._round_store(rng.standard_normal((w.T, w.n_h, w.d_c)).astype(np.float32) * 0.05, w.dtype)
    o_lat = dev(bits if w.dtype == "bf16" else vals, w.dtype)
    W_UV = store(x.weights["W_UV"], x.weights_bits.get("W_UV"), w.dtype)
    o = torch.full((w.T, w.n_h * w.d_h), float("nan"), device="cuda", dtype=o_lat.dtype)
    mla.mla_out_proj(dims_of(w, mla), o_lat, W_UV, o)
    assert mla.mla_get_device_error() == mla.MLA_OK
    ref = orc.out_proj(orc_dims_of(w, orc), vals, x.weights["W_UV"])
    assert_close(host(o), ref, "o")


def test_append_bad_position_reports_device_error(mla):
    import torch
    from tests.gpu_util import dev, dims_of, store
    w = CASES["v2_paged_T5"]
    x = synth.generate(w, seed=103)
    W = _weights(x, w.dtype)
    cache_t = dev(x.cache, w.dtype)
    before = cache_t.clone()
    cache = mla.Cache(cache_t, torch.from_numpy(x.block_table).cuda())
    pos = x.positions.copy()
    pos[0] = 1 << 20  # past the sequence's blocks
    mla.mla_cache_append(dims_of(w, mla), store(x.h, x.h_bits, w.dtype), W["W_DKV"], W["W_KR"],
                         torch.from_numpy(x.seq_idx).cuda(), torch.from_numpy(pos).cuda(), cache)
    assert mla.mla_get_device_error() == mla.MLA_ERR_DEVICE_DATA
    diff = (cache_t.view(torch.int16) != before.view(torch.int16)).any(dim=-1).sum().item()
    assert diff == w.T - 1  # every other row still written, the bad one skipped


def test_host_validation_rejects_bad_arguments(mla):
    import torch
    from tests.gpu_util import dims_of
    w = CASES["v2_paged_T5"]
    p = dims_of(w, mla)
    q = torch.zeros((1, 128, 576), device="cuda", dtype=torch.bfloat16)
    o = torch.zeros((1, 128, 512), device="cuda", dtype=torch.bfloat16)
    cache = mla.Cache(torch.zeros((2, 64, 576), device="cuda", dtype=torch.bfloat16),
                      torch.zeros((1, 2), dtype=torch.int32, device="cuda"))
    sl = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode(p, q, cache, sl, 0, o)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode(p, q[:, :, 1:], cache, sl, 1, o)  # misaligned base (2-byte offset)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode(p, q, cache, sl, 1, o, num_splits=-1)
    assert e.value.status == mla.MLA_ERR_INVALID_ARG
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode(p, q, cache, sl, 1, o, ws=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == mla.MLA_ERR_WORKSPACE
