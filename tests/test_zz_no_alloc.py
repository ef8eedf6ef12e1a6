"""mla_decode_noalloc (static library scratch) against mla_decode (caller
workspace): the same decode, compared element by element on two calls in a
row. Named so that pytest collects it last; it also passes on its own."""
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


def _inputs(mla, seq_lens, n_q=1):
    import torch
    from tests.gpu_util import dev, dims_of
    w = synth.shrink(synth.WORKLOADS["v2_b64_paged"], n_q=n_q)
    x = synth.generate_decode(w, 41, seq_lens=seq_lens)
    w = x.w
    p = dims_of(w, mla)
    q = dev(x.q_bits, "bf16")
    cache = mla.Cache(dev(x.cache, "bf16"), torch.from_numpy(x.block_table).cuda())
    sl = torch.from_numpy(x.seq_lens).cuda()
    return w, p, q, cache, sl


def _outputs(w):
    import torch
    T = w.B * w.n_q
    return (torch.full((T, w.n_h, w.d_c), float("nan"), device="cuda", dtype=torch.bfloat16),
            torch.full((T, w.n_h), float("nan"), device="cuda", dtype=torch.float32))


CASES = [
    (list(np.random.default_rng(42).integers(1, 3000, size=64)), 1),  # the 64-row limit, rows cut between clusters
    ([2, 65, 700, 4099, 257, 3], 2),
]


@pytest.mark.parametrize("overlap", [False, True])
@pytest.mark.parametrize("seq_lens,n_q", CASES)
def test_noalloc_matches_workspace_decode_twice(mla, seq_lens, n_q, overlap):
    """Two no-alloc calls enqueued back to back on one stream (with launch
    overlap on, the second call's decode may start while the first call's
    combine still reads the shared scratch), then one synchronisation."""
    from tests.gpu_util import assert_close, host
    w, p, q, cache, sl = _inputs(mla, seq_lens, n_q)
    ref_o, ref_l = _outputs(w)
    mla.mla_decode(p, q, cache, sl, n_q, ref_o, ref_l)
    assert mla.mla_get_device_error() == mla.MLA_OK
    was = mla.get_launch_overlap()
    mla.set_launch_overlap(overlap)
    try:
        outs = [_outputs(w) for _ in range(2)]
        for o, l in outs:
            mla.mla_decode_noalloc(p, q, cache, sl, n_q, o, l)
        assert mla.mla_get_device_error() == mla.MLA_OK
    finally:
        mla.set_launch_overlap(was)
    for o, l in outs:
        assert_close(host(o), host(ref_o), "o_lat (no-alloc vs workspace)")
        assert_close(host(l), host(ref_l), "lse (no-alloc vs workspace)")


def test_noalloc_matches_oracle(mla, orc):
    """The 64-row case against the fp64 oracle directly."""
    from tests.gpu_util import assert_close, host, orc_dims_of
    seq_lens, n_q = CASES[0]
    w0 = synth.shrink(synth.WORKLOADS["v2_b64_paged"], n_q=n_q)
    x = synth.generate_decode(w0, 41, seq_lens=seq_lens)
    w, p, q, cache, sl = _inputs(mla, seq_lens, n_q)
    o, l = _outputs(w)
    mla.mla_decode_noalloc(p, q, cache, sl, n_q, o, l)
    assert mla.mla_get_device_error() == mla.MLA_OK
    ref_o, ref_l = orc.decode(orc_dims_of(w, orc), x.q, orc.Cache(x.cache, x.block_table), x.seq_lens, n_q)
    assert_close(host(o), ref_o, "o_lat (no-alloc vs oracle)")
    assert_close(host(l), ref_l, "lse (no-alloc vs oracle)")


def test_noalloc_rejects_more_rows_than_its_scratch(mla):
    w, p, q, cache, sl = _inputs(mla, [100] * 33, n_q=2)  # 66 token rows > 64
    o, l = _outputs(w)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_noalloc(p, q, cache, sl, 2, o, l)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED
