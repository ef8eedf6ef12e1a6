"""GPU parity of order A, the training form (MLA walk-through, section 3 order
A: decompress K = [W_UK c_KV ; k_R] and V = W_UV c_KV per head, then the
ordinary 192-d attention), through the C ABI: mla_query_heads against the
oracle's per-head queries, and mla_attend_order_a against the oracle's order A
(all (token row, head) pairs on small cases, sampled pairs on multi-tile ones)
and against order B on the GPU (mla_decode then mla_out_proj, itself checked
against the oracle) element by element."""
import numpy as np
import pytest

from mla_latent_kv_33_b200 import synth

pytestmark = pytest.mark.gpu

V2 = synth.WORKLOADS["v2_b64_paged"]
TINY = synth.WORKLOADS["tiny_fp32"]


@pytest.fixture(scope="module")
def mla():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mla_latent_kv_33_b200 import mla as m
    return m


@pytest.mark.parametrize("name", ["v2_T5", "v2_T200", "tiny_fp32"])
def test_query_heads_match_oracle(mla, orc, name):
    import torch
    from tests.gpu_util import assert_close, dims_of, host, orc_dims_of, store
    w = {"v2_T5": synth.shrink(V2, B=5, L_lo=1, L_hi=100), "v2_T200": synth.shrink(V2, B=200, L_lo=1, L_hi=50),
         "tiny_fp32": TINY}[name]
    x = synth.generate(w, seed=107)
    p = dims_of(w, mla)
    W = {k: store(x.weights[k], x.weights_bits.get(k), w.dtype) for k in ("W_DQ", "W_UQ", "W_QR")}
    qa = torch.full((w.T, w.n_h, w.d_h + w.d_r), float("nan"), device="cuda",
                    dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32)
    mla.mla_query_heads(p, store(x.h, x.h_bits, w.dtype), W["W_DQ"], W["W_UQ"], W["W_QR"],
                        torch.from_numpy(x.positions).cuda(), qa)
    assert mla.mla_get_device_error() == mla.MLA_OK
    q, qc = orc.absorb_q(orc_dims_of(w, orc), x.h, x.weights["W_DQ"], x.weights["W_UQ"], x.weights["W_QR"],
                         x.weights["W_UK"], x.positions, want_qc=True)
    ref = np.concatenate([qc, q[:, :, w.d_c:]], axis=2)
    assert_close(host(qa), ref, "qa = [q_C | q_R]")


def _problem(w, seed, seq_lens, n_q):
    """Cache and lengths of the synthetic decode inputs; per-head queries and
    up-projections drawn here: qa ~ N(0, 0.5^2) (the spread of the scores
    matches the absorbed decode's), W_UK, W_UV ~ N(0, 1/d_c)."""
    x = synth.generate_decode(synth.shrink(w, n_q=n_q), seed, seq_lens=seq_lens)
    w = x.w
    rng = np.random.default_rng(seed + 1)
    qa, qa_bits = synth._round_store(rng.standard_normal((w.T, w.n_h, w.d_h + w.d_r)).astype(np.float32) * 0.5,
                                     w.dtype)
    W_UK, uk_bits = synth._round_store(rng.standard_normal((w.n_h * w.d_h, w.d_c)).astype(np.float32)
                                       / np.float32(np.sqrt(w.d_c)), w.dtype)
    W_UV, uv_bits = synth._round_store(rng.standard_normal((w.n_h * w.d_h, w.d_c)).astype(np.float32)
                                       / np.float32(np.sqrt(w.d_c)), w.dtype)
    return x, w, (qa, qa_bits), (W_UK, uk_bits), (W_UV, uv_bits)


def _run_order_a(mla, w, x, qa, uk, uv):
    import torch
    from tests.gpu_util import dev, dims_of, host
    p = dims_of(w, mla)
    cache = mla.Cache(dev(x.cache, w.dtype), None if x.block_table is None else torch.from_numpy(x.block_table).cuda())
    o = torch.full((w.T, w.n_h, w.d_h), float("nan"), device="cuda",
                   dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32)
    pick = (lambda v: dev(v[1], "bf16")) if w.dtype == "bf16" else (lambda v: dev(v[0], "fp32"))
    mla.mla_attend_order_a(p, pick(qa), pick(uk), pick(uv), cache, torch.from_numpy(x.seq_lens).cuda(), w.n_q, o)
    assert mla.mla_get_device_error() == mla.MLA_OK
    return host(o), cache, pick


ALL_PAIRS = {
    "v2_paged_nq1": (V2, 61, [1, 200, 333], 1),
    "v2_paged_nq7": (V2, 62, [64, 130], 7),
    "v2_contig_nq3": (synth.WORKLOADS["v2_b16_4k"], 63, [129, 70], 3),
    "tiny_fp32_nq1": (TINY, 64, [65], 1),
    "tiny_fp32_nq5": (TINY, 65, [9, 40], 5),
}


@pytest.mark.parametrize("case", list(ALL_PAIRS))
def test_order_a_matches_oracle_all_pairs(mla, orc, case):
    from tests.gpu_util import assert_close, orc_dims_of
    w0, seed, lens, n_q = ALL_PAIRS[case]
    x, w, qa, uk, uv = _problem(w0, seed, lens, n_q)
    got, _, _ = _run_order_a(mla, w, x, qa, uk, uv)
    po = orc_dims_of(w, orc)
    ref = orc.decode_order_a(po, qa[0][:, :, :w.d_h], qa[0][:, :, w.d_h:], uk[0], uv[0],
                             orc.Cache(x.cache, x.block_table), x.seq_lens, n_q)
    assert_close(got, ref, "o (order A)")


def test_order_a_two_query_blocks_sampled_and_equal_to_order_b(mla, orc):
    """130 new tokens per sequence (two blocks of query rows), contexts of
    several key tiles with ragged ends: sampled pairs against the oracle, every
    element against order B on the GPU with the same weights."""
    import torch
    from tests.gpu_util import assert_close, dev, dims_of, orc_dims_of, host
    n_q = 130
    x, w, qa, uk, uv = _problem(V2, 66, [700, 1000], n_q)
    got, cache, pick = _run_order_a(mla, w, x, qa, uk, uv)
    po = orc_dims_of(w, orc)
    rng = np.random.default_rng(9)
    rows = [0, 1, 127, 128, 129, 130, 257, 259] + rng.integers(0, w.T, 8).tolist()
    pairs = [(int(t), int(h)) for t in rows for h in rng.choice(w.n_h, 3, replace=False)]
    ref = orc.decode_order_a(po, qa[0][:, :, :w.d_h], qa[0][:, :, w.d_h:], uk[0], uv[0],
                             orc.Cache(x.cache, x.block_table), x.seq_lens, n_q, pairs=pairs)
    assert_close(np.stack([got[t, h] for t, h in pairs]), ref, "o (order A, sampled)")
    # order B with the same weights: q_lat,h = W_UK_h^T q_C,h (rounded once), decode, W_UV readout
    qc = qa[0][:, :, :w.d_h]
    q_lat = np.einsum("thi,hij->thj", qc, uk[0].reshape(w.n_h, w.d_h, w.d_c).astype(np.float64))
    qb, qb_bits = synth._round_store(np.concatenate([q_lat, qa[0][:, :, w.d_h:]], axis=2).astype(np.float32), "bf16")
    p = dims_of(w, mla)
    o_lat = torch.empty((w.T, w.n_h, w.d_c), device="cuda", dtype=torch.bfloat16)
    mla.mla_decode(p, dev(qb_bits, "bf16"), cache, torch.from_numpy(x.seq_lens).cuda(), n_q, o_lat)
    o_b = torch.empty((w.T, w.n_h * w.d_h), device="cuda", dtype=torch.bfloat16)
    mla.mla_out_proj(p, o_lat, pick(uv), o_b)
    assert mla.mla_get_device_error() == mla.MLA_OK
    assert_close(got.reshape(w.T, -1), host(o_b), "o: order A = order B")
