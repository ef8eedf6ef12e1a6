"""End-to-end parity of one decode step (append -> absorb -> decode -> out_proj)
on the five workloads, against the fp64 oracle.

Small cases compare every output element. Full-size cases run the exact
launch configuration bench.py times and compare sampled (token row, head)
outputs, which the oracle computes one by one; there the oracle's cache holds
its own appended rows rounded to the bf16 storage format.
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


def gpu_step(mla, x):
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
    return {"o_lat": host(o_lat), "lse": host(lse), "o": host(o), "q": host(q),
            "cache": cache_host(cache_t, w.dtype)}


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


def oracle_sampled(orc, x, pairs):
    """Oracle outputs for sampled (t, h): o_lat, lse, o slice."""
    from tests.gpu_util import orc_dims_of
    w = x.w
    po = orc_dims_of(w, orc)
    rows = orc.append_rows(po, x.h, x.weights["W_DKV"], x.weights["W_KR"], x.positions)
    cache = x.cache.copy()
    oc = orc.Cache(cache, x.block_table)
    flat = oc.data.reshape(-1, w.D)
    stored = synth.bf16_bits(rows.astype(np.float32)) if w.dtype == "bf16" else rows.astype(np.float32)
    for t in range(w.T):
        flat[oc.slot(int(x.seq_idx[t]), int(x.positions[t]))] = stored[t]
    ts = sorted({t for t, _ in pairs})
    q_rows = orc.absorb_q(po, x.h[ts], x.weights["W_DQ"], x.weights["W_UQ"], x.weights["W_QR"],
                          x.weights["W_UK"], x.positions[ts])
    q = np.zeros((w.T, w.n_h, w.D))
    q[ts] = q_rows
    o_lat, lse = orc.decode(po, q, oc, x.seq_lens, w.n_q, pairs=pairs)
    W_UV = x.weights["W_UV"].astype(np.float64)
    o = np.stack([W_UV[h * w.d_h:(h + 1) * w.d_h] @ o_lat[k] for k, (_, h) in enumerate(pairs)])
    return o_lat, lse, o


def _pairs(w, seq_lens, n=40, seed=0):
    rng = np.random.default_rng(seed)
    L = np.asarray(seq_lens)
    bs = {int(np.argmax(L)), int(np.argmin(L))}
    bs |= set(rng.integers(0, w.B, size=max(0, n // 4 - len(bs))).tolist())
    pairs = []
    for b in sorted(bs):
        for j in range(w.n_q):
            for h in rng.choice(w.n_h, size=4, replace=False):
                pairs.append((b * w.n_q + j, int(h)))
    return pairs


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
def test_full_size_step_sampled(mla, orc, name):
    from tests.gpu_util import assert_close
    w = synth.WORKLOADS[name]
    x = synth.generate(w)
    res = gpu_step(mla, x)
    pairs = _pairs(w, x.seq_lens)
    o_lat, lse, o = oracle_sampled(orc, x, pairs)
    assert_close(np.stack([res["o_lat"][t, h] for t, h in pairs]), o_lat, "o_lat (sampled)")
    assert_close(np.array([res["lse"][t, h] for t, h in pairs]), lse, "lse (sampled)")
    assert_close(np.stack([res["o"][t, h * w.d_h:(h + 1) * w.d_h] for t, h in pairs]), o, "o (sampled)")
    assert np.isfinite(res["o"]).all() and np.isfinite(res["o_lat"]).all()
