"""GPU parity of mla_decode against the fp64 oracle (order B), element by element.

Inputs are the seeded synthetic q and cache of synth.generate_decode; both
sides read the same bf16 values. Tolerance: |gpu - ref| <= 1e-2 + 1e-2 |ref|
on o_lat and lse. Unused cache slots hold NaN canaries, so any read past a
sequence's end would show up as a NaN in the output.
"""
import numpy as np
import pytest

from mla_latent_kv_33_b200 import synth

pytestmark = pytest.mark.gpu

V2 = synth.WORKLOADS["v2_b64_paged"]


@pytest.fixture(scope="module")
def mla():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mla_latent_kv_33_b200 import mla as m
    return m


def _run(mla, orc, w, seed, seq_lens, n_q=1, check_lse=True, pairs=None, num_splits=0):
    import torch
    from tests.gpu_util import assert_close, dev, dims_of, orc_dims_of, host
    w = synth.shrink(w, n_q=n_q)
    x = synth.generate_decode(w, seed, seq_lens=seq_lens)
    w = x.w
    p = dims_of(w, mla)
    q = dev(x.q_bits if w.dtype == "bf16" else x.q, w.dtype)
    cache_t = dev(x.cache, w.dtype)
    bt = None if x.block_table is None else torch.from_numpy(x.block_table).cuda()
    cache = mla.Cache(cache_t, bt)
    sl = torch.from_numpy(x.seq_lens).cuda()
    T = w.T
    o_lat = torch.full((T, w.n_h, w.d_c), float("nan"), device="cuda",
                       dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32)
    lse = torch.full((T, w.n_h), float("nan"), device="cuda", dtype=torch.float32)
    mla.mla_decode(p, q, cache, sl, n_q, o_lat, lse, num_splits=num_splits)
    assert mla.mla_get_device_error() == mla.MLA_OK
    oc = orc.Cache(x.cache, x.block_table)
    po = orc_dims_of(w, orc)
    if pairs is None:
        ref_o, ref_l = orc.decode(po, x.q, oc, x.seq_lens, n_q)
        assert_close(host(o_lat), ref_o, "o_lat")
        if check_lse:
            assert_close(host(lse), ref_l, "lse")
    else:
        ref_o, ref_l = orc.decode(po, x.q, oc, x.seq_lens, n_q, pairs=pairs)
        go, gl = host(o_lat), host(lse)
        assert_close(np.stack([go[t, h] for t, h in pairs]), ref_o, "o_lat (sampled)")
        assert_close(np.array([gl[t, h] for t, h in pairs]), ref_l, "lse (sampled)")
    return x


def test_decode_uses_tensor_cores_for_deepseek_dims(mla):
    from tests.gpu_util import dims_of
    assert mla.uses_tensor_cores(dims_of(V2, mla), mla.OP_DECODE)
    assert not mla.uses_tensor_cores(dims_of(synth.WORKLOADS["tiny_fp32"], mla), mla.OP_DECODE)


@pytest.mark.parametrize("seq_lens", [[1], [64], [65], [256], [257],
                                      [1, 2, 63, 64, 65, 127, 128, 129, 200, 1000],
                                      [191, 192, 193, 255, 256, 257, 300, 511, 512, 513, 700, 769]])
def test_decode_tc_paged_ragged(mla, orc, seq_lens):
    _run(mla, orc, V2, 11, seq_lens)


def test_decode_tc_paged_block_128(mla, orc):
    # blocks of 128 tokens: two 64-token value chunks per block
    _run(mla, orc, synth.shrink(V2, block_size=128), 22, [1, 129, 300, 1000])


def test_decode_tc_contiguous(mla, orc):
    w = synth.shrink(synth.WORKLOADS["v2_b16_4k"])
    _run(mla, orc, w, 12, [700, 33, 1500, 64])
    _run(mla, orc, w, 21, [257, 1, 511, 130])


def test_decode_tc_splits_long_sequences(mla, orc):
    # few long rows: every row is cut into many pieces and merged by the combine
    _run(mla, orc, V2, 13, [5000, 4099, 3001])


def test_decode_tc_many_short_sequences(mla, orc):
    # more rows than clusters: several rows per cluster, most finished in place
    rng = np.random.default_rng(14)
    _run(mla, orc, V2, 14, list(rng.integers(1, 300, size=300)))


# Split-KV independence: forced split counts S (each token row cut into
# min(S, its tiles) pieces, merged by the log-sum-exp combine) and the
# automatic plan (S = 0) all match the oracle.
SPLIT_LENS = [3000, 1, 700, 5000, 257, 64, 1800]


@pytest.mark.parametrize("splits", [1, 2, 7, 0])
def test_decode_tc_split_independence(mla, orc, splits):
    _run(mla, orc, V2, 23, SPLIT_LENS, num_splits=splits)


@pytest.mark.parametrize("splits", [3, 74])
def test_decode_tc_forced_splits_two_queries(mla, orc, splits):
    # 74 pieces ask for more than the tiles of every row here: one tile per piece
    _run(mla, orc, V2, 24, [2, 513, 4000, 9000], n_q=2, num_splits=splits)


def test_decode_tc_forced_splits_long_rows(mla, orc):
    # long rows cut into more pieces than there are clusters
    _run(mla, orc, V2, 25, [30000, 20011], num_splits=200)


def test_decode_tc_two_queries_causal(mla, orc):
    _run(mla, orc, V2, 15, [2, 64, 65, 66, 1000, 3000], n_q=2)


# n_q > 1 runs the kernel whose clusters form one group per query position,
# each group cutting its own line of rows (rows ordered by query position).
@pytest.mark.parametrize("n_q, seq_lens", [
    (3, [3, 257, 4000, 9000, 700]),           # three groups; two clusters left over (74 = 3 x 24 + 2)
    (2, [5000, 4099, 3001, 12000]),            # long rows cut across the clusters of each group
    (4, [4, 300, 2000, 65, 128, 129, 6000]),   # four groups, ragged tiles at every edge
])
def test_decode_tc_query_position_groups(mla, orc, n_q, seq_lens):
    _run(mla, orc, V2, 26 + n_q, seq_lens, n_q=n_q)


def test_decode_tc_query_position_groups_many_rows(mla, orc):
    # more rows than clusters in every group: rows finished in place and cut
    rng = np.random.default_rng(30)
    _run(mla, orc, V2, 30, list(rng.integers(2, 900, size=160)), n_q=2)


def test_decode_tc_bigger_scores_rescale(mla, orc):
    # larger query spread makes the running max move by more than 2^8 and
    # exercises the rescaling of the accumulator
    import torch  # noqa: F401
    w = V2
    x = synth.generate_decode(w, 16, seq_lens=[2500, 777])
    x.q[:] *= 6.0
    # re-round to bf16 after scaling (exact: powers of two and 3 keep within range)
    x.q_bits[:] = synth.bf16_bits(x.q)
    x.q[:] = synth.bf16_to_f32(x.q_bits)
    from tests.gpu_util import assert_close, dev, dims_of, orc_dims_of, host
    p = dims_of(w, mla)
    q = dev(x.q_bits, "bf16")
    bt = torch.from_numpy(x.block_table).cuda()
    cache = mla.Cache(dev(x.cache, "bf16"), bt)
    sl = torch.from_numpy(x.seq_lens).cuda()
    o_lat = torch.empty((2, 128, 512), device="cuda", dtype=torch.bfloat16)
    lse = torch.empty((2, 128), device="cuda", dtype=torch.float32)
    mla.mla_decode(p, q, cache, sl, 1, o_lat, lse)
    assert mla.mla_get_device_error() == mla.MLA_OK
    ref_o, ref_l = orc.decode(orc_dims_of(w, orc), x.q, orc.Cache(x.cache, x.block_table), x.seq_lens, 1)
    assert_close(host(o_lat), ref_o, "o_lat")
    assert_close(host(lse), ref_l, "lse")


def test_decode_simt_generic_dims_bf16(mla, orc):
    w = synth.Workload("small", 0, d=64, n_h=3, d_h=16, d_c=48, d_cq=32, d_r=8, B=1, n_q=1,
                       lens="fixed", L=1, paged=True, block_size=16)
    _run(mla, orc, w, 17, [1, 15, 16, 17, 100], n_q=1)
    _run(mla, orc, w, 18, [2, 40], n_q=2)


def test_decode_simt_fp32_contiguous(mla, orc):
    w = synth.WORKLOADS["tiny_fp32"]
    _run(mla, orc, w, 19, [65, 3, 130])


def test_decode_bad_seq_len_reports_device_error(mla):
    import torch
    from tests.gpu_util import dev, dims_of
    x = synth.generate_decode(V2, 20, seq_lens=[100, 70])
    p = dims_of(V2, mla)
    bt = torch.from_numpy(x.block_table).cuda()
    cache = mla.Cache(dev(x.cache, "bf16"), bt)
    sl = torch.tensor([100, 10_000], dtype=torch.int32, device="cuda")  # second exceeds capacity
    o = torch.zeros((2, 128, 512), device="cuda", dtype=torch.bfloat16)
    mla.mla_decode(p, dev(x.q_bits, "bf16"), cache, sl, 1, o)
    assert mla.mla_get_device_error() == mla.MLA_ERR_DEVICE_DATA
    assert mla.mla_get_device_error() == mla.MLA_OK  # the word is cleared on read
    assert torch.all(o[1] == 0)  # the bad row was left unwritten
