"""Launch overlap (programmatic dependent launch) changes when kernels start,
never what they compute: the whole step (append -> absorb -> decode ->
out_proj) on the full-size paged workload gives bit-identical outputs with
overlap off, with it on, and replayed from a CUDA graph captured with it on
(the way bench.py times the step)."""
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


def _setup(mla, name):
    import torch
    w = synth.WORKLOADS[name]
    x = synth.generate(w)
    assert w.dtype == "bf16"
    bf = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()
    W = {k: bf(x.weights_bits[k]) for k in x.weights_bits}
    cache0 = bf(x.cache)  # bf16 workloads keep the cache as its storage bits
    bt = torch.from_numpy(x.block_table).cuda() if x.block_table is not None else None
    p = mla.dims(w.d, w.n_h, w.d_h, w.d_c, w.d_cq, w.d_r, w.rope_base, 0.0, w.dtype)
    T = w.T
    s = {
        "w": w, "p": p, "W": W, "cache0": cache0, "bt": bt,
        "cache_t": cache0.clone(),
        "h": bf(x.h_bits), "pos": torch.from_numpy(x.positions).cuda(),
        "sidx": torch.from_numpy(x.seq_idx).cuda(), "sl": torch.from_numpy(x.seq_lens).cuda(),
        "q": torch.empty((T, w.n_h, w.D), device="cuda", dtype=torch.bfloat16),
        "o_lat": torch.empty((T, w.n_h, w.d_c), device="cuda", dtype=torch.bfloat16),
        "lse": torch.empty((T, w.n_h), device="cuda", dtype=torch.float32),
        "o": torch.empty((T, w.n_h * w.d_h), device="cuda", dtype=torch.bfloat16),
    }
    s["cache"] = mla.Cache(s["cache_t"], bt)
    s["ws"] = {op: torch.empty(max(1, mla.workspace_size(p, op, w.B if op == mla.OP_DECODE else T, w.n_q)),
                               dtype=torch.uint8, device="cuda")
               for op in (mla.OP_APPEND, mla.OP_ABSORB, mla.OP_DECODE, mla.OP_OUT_PROJ)}
    return s


def _step(mla, s, stream):
    p, W, ws, w = s["p"], s["W"], s["ws"], s["w"]
    mla.mla_cache_append(p, s["h"], W["W_DKV"], W["W_KR"], s["sidx"], s["pos"], s["cache"],
                         ws=ws[mla.OP_APPEND], stream=stream)
    mla.mla_absorb_q(p, s["h"], W["W_DQ"], W["W_UQ"], W["W_QR"], W["W_UK"], s["pos"], s["q"],
                     ws=ws[mla.OP_ABSORB], stream=stream)
    mla.mla_decode(p, s["q"], s["cache"], s["sl"], w.n_q, s["o_lat"], s["lse"], ws=ws[mla.OP_DECODE],
                   stream=stream)
    mla.mla_out_proj(p, s["o_lat"], W["W_UV"], s["o"], ws=ws[mla.OP_OUT_PROJ], stream=stream)


def _results(s):
    """Host copies as raw bits (the cache keeps NaN canaries, which compare
    unequal as floating point)."""
    import torch
    bits = {torch.bfloat16: torch.int16, torch.float32: torch.int32}
    return {k: s[k].detach().cpu().view(bits[s[k].dtype]).clone() for k in ("q", "o_lat", "lse", "o", "cache_t")}


def _clear(s):
    s["cache_t"].copy_(s["cache0"])
    for k in ("q", "o_lat", "o"):
        s[k].zero_()
    s["lse"].fill_(float("nan"))
    import torch
    torch.cuda.synchronize()  # the step runs on its own stream


# v2_b64_paged: the bench step (fused per-head absorb); v3_b128_nq2: 256 token
# rows, where the absorb runs as separate GEMMs (MN-major W_UK operand)
@pytest.mark.parametrize("name", ["v2_b64_paged", "v3_b128_nq2"])
def test_overlap_gives_identical_results_eager_and_in_a_graph(mla, name):
    import torch
    s = _setup(mla, name)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    try:
        mla.set_launch_overlap(False)
        with torch.cuda.stream(stream):
            _step(mla, s, stream)
        torch.cuda.synchronize()
        assert mla.mla_get_device_error() == mla.MLA_OK
        ref = _results(s)

        mla.set_launch_overlap(True)
        for _ in range(2):
            _clear(s)
            with torch.cuda.stream(stream):
                _step(mla, s, stream)
            torch.cuda.synchronize()
            assert mla.mla_get_device_error() == mla.MLA_OK
            got = _results(s)
            for k in ref:
                assert torch.equal(got[k], ref[k]), f"{k} differs with launch overlap (eager)"

        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            _step(mla, s, stream)
        for _ in range(3):
            _clear(s)
            with torch.cuda.stream(stream):
                g.replay()
            torch.cuda.synchronize()
            assert mla.mla_get_device_error() == mla.MLA_OK
            got = _results(s)
            for k in ref:
                assert torch.equal(got[k], ref[k]), f"{k} differs with launch overlap (graph replay)"
        del g
    finally:
        mla.set_launch_overlap(False)
