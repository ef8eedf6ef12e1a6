"""End-to-end parity of one decode step (append -> absorb -> decode -> out_proj)
on the five workloads, against the fp64 oracle, element by element.

Small cases run the oracle's whole chain in fp64. Full-size cases run the
workloads at the sizes bench.py times, through the same calls, and compare
every element of o_lat, lse and o; there the oracle's cache keeps its own
appended rows rounded once to the bf16 storage format (the cache is a
storage point), and its q, o_lat and o stay in fp64.
"""
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


def gpu_step(mla, x, want_cache=True):
    """Run the hot path through the C ABI; return host copies of the results."""
    import torch
    from tests.gpu_util import cache_host, dev, dims_of, host, store
    w = x.w
    p = dims_of(w, mla)
    W = {k: store(x.weights[k], x.weights_bits.get(k), w.dtype) for k in x.weights}
    cache_t = dev(x.cache, w.dtype)
    bt = None if x.block_table is None else torch.from_numpy(x.block_table).cuda()
    cache = mla.Cache(cache_t, bt)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    if x.prefill_h is not None:   # build the earlier context through the same append
        ph = dev(x.prefill_h, w.dtype) if w.dtype == "fp32" else dev(synth.bf16_bits(x.prefill_h), w.dtype)
        mla.mla_cache_append(p, ph, W["W_DKV"], W["W_KR"], torch.from_numpy(x.prefill_seq).cuda(),
                             torch.from_numpy(x.prefill_pos).cuda(), cache)
    h = store(x.h, x.h_bits, w.dtype)
    pos = torch.from_numpy(x.positions).cuda()
    mla.mla_cache_append(p, h, W["W_DKV"], W["W_KR"], torch.from_numpy(x.seq_idx).cuda(), pos, cache)
    q = torch.empty((w.T, w.n_h, w.D), device="cuda", dtype=tdt)
    mla.mla_absorb_q(p, h, W["W_DQ"], W["W_UQ"], W["W_QR"], W["W_UK"], pos, q)
    o_lat = torch.empty((w.T, w.n_h, w.d_c), device="cuda", dtype=tdt)
    lse = torch.empty((w.T, w.n_h), device="cuda", dtype=torch.float32)
    mla.mla_decode(p, q, cache, torch.from_numpy(x.seq_lens).cuda(), w.n_q, o_lat, lse)
    o = torch.empty((w.T, w.n_h * w.d_h), device="cuda", dtype=tdt)
    mla.mla_out_proj(p, o_lat, W["W_UV"], o)
    assert mla.mla_get_device_error() == mla.MLA_OK
    out = {"o_lat": host(o_lat), "lse": host(lse), "o": host(o), "q": host(q)}
    if want_cache:
        out["cache"] = cache_host(cache_t, w.dtype)
    return out


def oracle_full(orc, x):
    from tests.gpu_util import orc_dims_of
    w = x.w
    po = orc_dims_of(w, orc)
    cache = x.cache.copy()
    if x.prefill_h is not None:
        rows = orc.append_rows(po, x.prefill_h, x.weights["W_DKV"], x.weights["W_KR"], x.prefill_pos)
        c64 = orc.Cache(cache.astype(np.float64) if cache.dtype == np.float32 else cache, x.block_table)
        flat = c64.data.reshape(-1, w.D)
        for i in range(rows.shape[0]):
            flat[c64.slot(int(x.prefill_seq[i]), int(x.prefill_pos[i]))] = rows[i]
        before = c64
    else:
        before = orc.Cache(cache, x.block_table)
    return orc.step(po, x.weights, x.h, x.positions, x.seq_idx, before, x.seq_lens, w.n_q)


def oracle_full_size(orc, x):
    """The oracle's own chain over the whole workload: its appended rows
    (rounded once to bf16 where the cache stores them), the absorbed queries,
    order-B decode of every (token row, head) and the W_UV readout, in fp64."""
    from tests.gpu_util import orc_dims_of
    w = x.w
    po = orc_dims_of(w, orc)
    rows = orc.append_rows(po, x.h, x.weights["W_DKV"], x.weights["W_KR"], x.positions)
    oc = orc.Cache(x.cache.copy(), x.block_table)
    flat = oc.data.reshape(-1, w.D)
    for t in range(w.T):
        flat[oc.slot(int(x.seq_idx[t]), int(x.positions[t]))] = synth.bf16_bits(rows[t].astype(np.float32))
    q = orc.absorb_q(po, x.h, x.weights["W_DQ"], x.weights["W_UQ"], x.weights["W_QR"], x.weights["W_UK"],
                     x.positions)
    o_lat, lse = orc.decode(po, q, oc, x.seq_lens, w.n_q)
    o = orc.out_proj(po, o_lat, x.weights["W_UV"])
    return {"o_lat": o_lat, "lse": lse, "o": o}


def _check_full(res, ref, w):
    from tests.gpu_util import assert_close
    assert_close(res["o_lat"], ref["o_lat"], "o_lat")
    assert_close(res["lse"], ref["lse"], "lse")
    assert_close(res["o"], ref["o"], "o")


def test_tiny_fp32_step(mla, orc):
    w = synth.WORKLOADS["tiny_fp32"]
    x = synth.generate(w)
    _check_full(gpu_step(mla, x), oracle_full(orc, x), w)


SMALL = {
    "v2_b16_4k": dict(B=4),
    "v2_b64_paged": dict(B=6, L_lo=1, L_hi=2000),
    "v2_b4_128k": dict(B=2, L=3000),
    "v3_b128_nq2": dict(B=5, L_lo=2, L_hi=1500, median=300.0),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_step_all_elements(mla, orc, name):
    w = synth.shrink(synth.WORKLOADS[name], **SMALL[name])
    x = synth.generate(w)
    _check_full(gpu_step(mla, x), oracle_full(orc, x), w)


@pytest.mark.parametrize("name", ["v2_b16_4k", "v2_b64_paged", "v2_b4_128k", "v3_b128_nq2"])
def test_full_size_step_all_elements(mla, orc, name):
    w = synth.WORKLOADS[name]
    x = synth.generate(w)
    res = gpu_step(mla, x, want_cache=False)
    assert np.isfinite(res["o"]).all() and np.isfinite(res["o_lat"]).all()
    _check_full(res, oracle_full_size(orc, x), w)
