"""Host-side validation of the C ABI, on CPU. Each call below is rejected
before it touches the device, so the fake (never dereferenced) pointers it
receives are safe: the tests pin the status, and the message that
mla_last_error_message reports for it."""
import ctypes as C

import pytest

torch = pytest.importorskip("torch")
# The fake pointers below must never reach a kernel. Every call is built to be
# rejected first, but this module runs only where no device is visible, so a
# check that moved behind a launch could not turn into a memory fault.
pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="host-only checks with fake device pointers")


@pytest.fixture(scope="module")
def m():
    from mla_latent_kv_33_b200 import build
    build.build()
    from mla_latent_kv_33_b200 import mla
    return mla


A = 0x10000          # a 16-byte aligned address that is never dereferenced
MIS = 0x10008        # 8-byte aligned only


def v2(m, **kw):
    args = dict(d=5120, n_h=128, d_h=128, d_c=512, d_cq=1536, d_r=64, rope_base=10000.0, softmax_scale=0.0,
                dtype="bf16")
    args.update(kw)
    return m.dims(**args)


def paged_cache(m, **kw):
    c = m.CacheDesc(A, 1, 64, A, 128, 64, 0, 4096)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def last_msg(m):
    return m._lib.mla_last_error_message().decode()


def append(m, d, h=A, T=64, cache=None, ws=A, ws_bytes=1 << 30):
    cache = cache if cache is not None else paged_cache(m)
    return m._lib.mla_cache_append(C.byref(d), h, A, A, A, A, T, C.byref(cache), ws, ws_bytes, None)


def decode(m, d, B=64, n_q=1, q=A, o_lat=A, cache=None, num_splits=0, ws=A, ws_bytes=1 << 30):
    cache = cache if cache is not None else paged_cache(m)
    return m._lib.mla_decode(C.byref(d), q, C.byref(cache), A, B, n_q, o_lat, A, num_splits, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status,words", [
    (dict(n_h=0), "MLA_ERR_INVALID_ARG", "positive"),
    (dict(d_r=63), "MLA_ERR_INVALID_ARG", "even"),
    (dict(rope_base=1.0), "MLA_ERR_INVALID_ARG", "rope_base"),
    (dict(d_c=1000, d_r=64), "MLA_ERR_UNSUPPORTED", "1024"),
])
def test_dims_are_checked_first(m, kw, status, words):
    s = append(m, v2(m, **kw))
    assert s == getattr(m, status)
    assert words in last_msg(m)


def test_bad_dtype(m):
    d = v2(m)
    d.dtype = 7
    assert append(m, d) == m.MLA_ERR_INVALID_ARG and "dtype" in last_msg(m)


def test_null_dims(m):
    s = m._lib.mla_cache_append(None, A, A, A, A, A, 64, C.byref(paged_cache(m)), A, 1 << 30, None)
    assert s == m.MLA_ERR_INVALID_ARG and "NULL" in last_msg(m)


def test_append_arguments(m):
    d = v2(m)
    assert append(m, d, T=0) == m.MLA_ERR_INVALID_ARG and "T must be positive" in last_msg(m)
    assert append(m, d, h=None) == m.MLA_ERR_INVALID_ARG and "NULL" in last_msg(m)
    assert append(m, d, h=MIS) == m.MLA_ERR_INVALID_ARG and "aligned" in last_msg(m)
    assert append(m, d, cache=paged_cache(m, block_table=None)) == m.MLA_ERR_INVALID_ARG
    assert "block_table" in last_msg(m)
    assert append(m, d, cache=paged_cache(m, data=MIS)) == m.MLA_ERR_INVALID_ARG
    assert append(m, d, cache=m.CacheDesc(A, 0, 0, None, 0, 4, 0, 0)) == m.MLA_ERR_INVALID_ARG
    assert "max_len" in last_msg(m)
    need = m._lib.mla_workspace_size(C.byref(d), m.OP_APPEND, 64, 1, 0, 0)
    assert need > 0
    assert append(m, d, ws_bytes=need - 1) == m.MLA_ERR_WORKSPACE and str(need) in last_msg(m)
    assert append(m, d, ws=None, ws_bytes=need) == m.MLA_ERR_WORKSPACE


def test_absorb_and_out_proj_arguments(m):
    d = v2(m)
    ab = m._lib.mla_absorb_q
    assert ab(C.byref(d), A, A, A, A, A, A, 64, MIS, A, 1 << 30, None) == m.MLA_ERR_INVALID_ARG
    assert ab(C.byref(d), A, A, A, A, None, A, 64, A, A, 1 << 30, None) == m.MLA_ERR_INVALID_ARG
    need = m._lib.mla_workspace_size(C.byref(d), m.OP_ABSORB, 64, 1, 0, 0)
    assert need > 0
    assert ab(C.byref(d), A, A, A, A, A, A, 64, A, A, need - 1, None) == m.MLA_ERR_WORKSPACE
    op = m._lib.mla_out_proj
    assert op(C.byref(d), A, A, 0, A, A, 1 << 30, None) == m.MLA_ERR_INVALID_ARG
    assert op(C.byref(d), MIS, A, 64, A, A, 1 << 30, None) == m.MLA_ERR_INVALID_ARG
    # the tensor-core out-projection needs no workspace (one CTA per head, no split-K)
    assert m._lib.mla_workspace_size(C.byref(d), m.OP_OUT_PROJ, 64, 1, 0, 0) == 0
    need = m._lib.mla_workspace_size(C.byref(v2(m, dtype="fp32")), m.OP_OUT_PROJ, 64, 1, 0, 0)
    assert need > 0  # the CUDA-core path keeps fp32 intermediate rows
    assert op(C.byref(v2(m, dtype="fp32")), A, A, 64, A, A, need - 1, None) == m.MLA_ERR_WORKSPACE


def test_o_proj_arguments(m):
    d = v2(m)
    op = m._lib.mla_o_proj
    assert op(C.byref(d), A, A, 0, A, A, 1 << 30, None) == m.MLA_ERR_INVALID_ARG
    assert op(C.byref(d), A, None, 64, A, A, 1 << 30, None) == m.MLA_ERR_INVALID_ARG
    assert op(C.byref(d), A, A, 64, MIS, A, 1 << 30, None) == m.MLA_ERR_INVALID_ARG and "aligned" in last_msg(m)
    need = m._lib.mla_workspace_size(C.byref(d), m.OP_O_PROJ, 64, 1, 0, 0)
    assert 0 < need < 1 << 30  # split-K fp32 partials of the 5120 x 64 output
    assert op(C.byref(d), A, A, 64, A, A, need - 1, None) == m.MLA_ERR_WORKSPACE


def test_decode_arguments(m):
    d = v2(m)
    assert decode(m, d, B=0) == m.MLA_ERR_INVALID_ARG
    assert decode(m, d, n_q=0) == m.MLA_ERR_INVALID_ARG
    assert decode(m, d, q=None) == m.MLA_ERR_INVALID_ARG
    assert decode(m, d, o_lat=MIS) == m.MLA_ERR_INVALID_ARG and "aligned" in last_msg(m)
    assert decode(m, d, B=65) == m.MLA_ERR_INVALID_ARG and "num_seqs" in last_msg(m)
    assert decode(m, d, num_splits=-1) == m.MLA_ERR_INVALID_ARG
    need = m._lib.mla_workspace_size(C.byref(d), m.OP_DECODE, 64, 1, 0, 0)
    assert 0 < need < 1 << 30
    assert decode(m, d, ws_bytes=need - 1) == m.MLA_ERR_WORKSPACE
    # forced splits: partials for min(S, tiles of the longest row the cache holds) pieces of every row;
    # the paged cache here holds 128 blocks of 64 = 8192 tokens = 32 tiles per row
    cap = 128 * 64
    need4 = m._lib.mla_workspace_size(C.byref(d), m.OP_DECODE, 64, 1, cap, 4)
    need64 = m._lib.mla_workspace_size(C.byref(d), m.OP_DECODE, 64, 1, cap, 64)
    assert need64 > need4 >= need
    assert need64 == m._lib.mla_workspace_size(C.byref(d), m.OP_DECODE, 64, 1, cap, 32)  # capped at 32 tiles
    assert m._lib.mla_workspace_size(C.byref(d), m.OP_DECODE, 64, 1, 0, 64) > need64      # unknown length: 64 per row
    assert decode(m, d, num_splits=64, ws_bytes=need64 - 1) == m.MLA_ERR_WORKSPACE


def test_noalloc_decode_limit(m):
    d = v2(m)
    c = paged_cache(m, num_seqs=128)
    s = m._lib.mla_decode_noalloc(C.byref(d), A, C.byref(c), A, 33, 2, A, A, None)
    assert s == m.MLA_ERR_UNSUPPORTED and "66" in last_msg(m)


def test_workspace_sizes(m):
    d = v2(m)
    ws = lambda op, rows, n_q=1: m._lib.mla_workspace_size(C.byref(d), op, rows, n_q, 0, 0)
    # decode: a plan plus fp32 partials of 128 x 512 (and 128 lse) per slot,
    # slots = token rows + clusters; more rows never need less
    assert ws(m.OP_DECODE, 64) > 64 * 128 * 512 * 4
    assert ws(m.OP_DECODE, 128) > ws(m.OP_DECODE, 64)
    assert ws(m.OP_DECODE, 64, 2) > ws(m.OP_DECODE, 64, 1)
    assert ws(m.OP_DECODE, 0) == 0 and ws(m.OP_APPEND, -1) == 0
    assert m._lib.mla_workspace_size(None, m.OP_DECODE, 64, 1, 0, 0) == 0
    assert ws(99, 64) == 0  # unknown op


def test_tensor_core_geometry_switch(m):
    d = v2(m)
    assert all(m._lib.mla_uses_tensor_cores(C.byref(d), op) == 1 for op in range(5))
    assert m._lib.mla_uses_tensor_cores(C.byref(v2(m, dtype="fp32")), m.OP_DECODE) == 0
    assert m._lib.mla_uses_tensor_cores(C.byref(v2(m, n_h=64)), m.OP_DECODE) == 0
    assert m._lib.mla_uses_tensor_cores(C.byref(d), 99) == 0


def test_python_binding_raises_with_status_and_message(m):
    import torch
    d = v2(m)
    h = torch.zeros((0, 5120), dtype=torch.bfloat16)  # T = 0: rejected before any device work
    class NoStream:  # the call is rejected before it would use a stream
        cuda_stream = 0
    with pytest.raises(m.MlaError) as e:
        m.mla_absorb_q(d, h, h, h, h, h, torch.zeros(0, dtype=torch.int32), h, ws=None, stream=NoStream())
    assert e.value.status == m.MLA_ERR_INVALID_ARG
    assert "T must be positive" in str(e.value)


def test_next_row_entry_points_validate_before_any_launch(m):
    d = v2(m)
    c = paged_cache(m)
    L = m._lib
    # NULL tensors
    assert L.mla_absorb_wo(C.byref(d), None, A, A, None) == m.MLA_ERR_INVALID_ARG
    assert L.mla_absorb_merge(C.byref(d), A, None, A, None) == m.MLA_ERR_INVALID_ARG
    assert L.mla_o_proj_latent(C.byref(d), A, A, 4, None, A, 1 << 30, None) == m.MLA_ERR_INVALID_ARG
    # misaligned, non-positive T, too little workspace
    assert L.mla_absorb_wo(C.byref(d), MIS, A, A, None) == m.MLA_ERR_INVALID_ARG and "aligned" in last_msg(m)
    assert L.mla_o_proj_latent(C.byref(d), A, A, 0, A, A, 1 << 30, None) == m.MLA_ERR_INVALID_ARG
    need = L.mla_workspace_size(C.byref(d), m.OP_O_PROJ_LATENT, 8, 1, 0, 0)
    assert need > 0 and L.mla_o_proj_latent(C.byref(d), A, A, 8, A, A, need - 1, None) == m.MLA_ERR_WORKSPACE
    need = L.mla_workspace_size(C.byref(d), m.OP_ABSORB_MERGED, 8, 1, 0, 0)
    assert need > 0
    assert L.mla_absorb_q_merged(C.byref(d), A, A, A, A, A, 8, A, A, need - 1, None) == m.MLA_ERR_WORKSPACE
    assert L.mla_absorb_q_merged(C.byref(d), A, A, A, A, None, 8, A, A, need, None) == m.MLA_ERR_INVALID_ARG
    need = L.mla_workspace_size(C.byref(d), m.OP_FRONT_END, 8, 1, 0, 0)
    # the fused front end needs at least what the append and the absorb need
    assert need >= L.mla_workspace_size(C.byref(d), m.OP_ABSORB, 8, 1, 0, 0)
    assert L.mla_front_end(C.byref(d), A, A, A, A, A, A, A, A, A, 8, C.byref(c), A, A, need - 1,
                           None) == m.MLA_ERR_WORKSPACE
    assert L.mla_front_end(C.byref(d), A, A, A, A, A, A, A, A, A, 0, C.byref(c), A, A, need,
                           None) == m.MLA_ERR_INVALID_ARG
    bad = paged_cache(m, block_table=None)
    assert L.mla_front_end(C.byref(d), A, A, A, A, A, A, A, A, A, 8, C.byref(bad), A, A, need,
                           None) == m.MLA_ERR_INVALID_ARG and "block_table" in last_msg(m)
    # the self-test needs a positive limit and 64 KiB of aligned scratch
    assert L.mla_selftest_timeout(0, A, 65536, None) == m.MLA_ERR_INVALID_ARG
    assert L.mla_selftest_timeout(1000, A, 65535, None) == m.MLA_ERR_INVALID_ARG
    assert L.mla_selftest_timeout(1000, MIS, 65536, None) == m.MLA_ERR_INVALID_ARG
    # every new op is served by the tensor cores at DeepSeek dims
    assert all(L.mla_uses_tensor_cores(C.byref(d), op) == 1 for op in range(9))
