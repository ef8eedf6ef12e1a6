"""Pins for the fp64 oracle against facts fixed by the pages and by mathematics.

None of these checks re-runs the oracle's own formula: each one compares it to
a closed form worked out by hand, to a library routine (numpy / torch on CPU),
to an invariant the method must satisfy (order A == order B, RoPE relative
position, split-KV algebra, paged == contiguous), or to numbers printed on the
pages (tests/golden/).
"""
import json
import math
import os

import numpy as np
import pytest

from mla_latent_kv_33_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(rng, d=24, n_h=3, d_h=4, d_c=8, d_cq=10, d_r=4, B=2, n_q=1, lens=(5, 9)):
    w = {
        "W_DKV": rng.standard_normal((d_c, d)) / math.sqrt(d),
        "W_KR": rng.standard_normal((d_r, d)) / math.sqrt(d),
        "W_DQ": rng.standard_normal((d_cq, d)) / math.sqrt(d),
        "W_UQ": rng.standard_normal((n_h * d_h, d_cq)) / math.sqrt(d_cq),
        "W_QR": rng.standard_normal((n_h * d_r, d_cq)) / math.sqrt(d_cq),
        "W_UK": rng.standard_normal((n_h * d_h, d_c)) / math.sqrt(d_c),
        "W_UV": rng.standard_normal((n_h * d_h, d_c)) / math.sqrt(d_c),
    }
    seq_lens = np.array(lens, np.int32)
    return w, seq_lens, dict(d=d, n_h=n_h, d_h=d_h, d_c=d_c, d_cq=d_cq, d_r=d_r)


def _build_cache_by_append(orc, p, w, rng, seq_lens, shift=0, hs=None):
    """Fill a contiguous fp64 cache by running the oracle's own append at
    positions 0..L-1 (+shift); returns (cache, hs)."""
    B = len(seq_lens)
    L = int(seq_lens.max())
    D = p.d_c + p.d_r
    cache = np.full((B, L, D), np.nan)
    if hs is None:
        hs = [rng.standard_normal((int(seq_lens[b]), p.d)) for b in range(B)]
    for b in range(B):
        pos = np.arange(int(seq_lens[b]), dtype=np.int32) + shift
        cache[b, : seq_lens[b]] = orc.append_rows(p, hs[b], w["W_DKV"], w["W_KR"], pos)
    return cache, hs


# ---------------------------------------------------------------- RoPE ----

def test_rope_d2_closed_form(orc):
    # d_R = 2, one pair, theta_0 = base^0 = 1: rotation by the position angle.
    for pos in (1.0, 2.5, -0.7):
        assert np.allclose(orc.rope([1.0, 0.0], pos), [math.cos(pos), math.sin(pos)], atol=1e-15)
        assert np.allclose(orc.rope([0.0, 1.0], pos), [-math.sin(pos), math.cos(pos)], atol=1e-15)


def test_rope_frequencies_and_interleaved_pairs(orc):
    # d_R = 4, base 10000: pair i=1 rotates by pos * 10000^(-2/4) = pos / 100,
    # and pairs are (0,1),(2,3) (RoFormer interleaving), so a unit vector on
    # coordinate 2 moves only into coordinate 3.
    out = orc.rope([0.0, 0.0, 1.0, 0.0], 3.0)
    assert np.allclose(out, [0, 0, math.cos(0.03), math.sin(0.03)], atol=1e-15)
    out = orc.rope([1.0, 0.0, 0.0, 0.0], 3.0)
    assert np.allclose(out, [math.cos(3.0), math.sin(3.0), 0, 0], atol=1e-15)


def test_rope_identity_norm_and_relative_position(orc):
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    assert np.array_equal(orc.rope(q, 0.0), q)
    for m, n in ((5, 3), (131071, 17), (100, 100)):
        assert abs(np.linalg.norm(orc.rope(q, m)) - np.linalg.norm(q)) < 1e-12
        a = orc.rope(q, m) @ orc.rope(k, n)
        delta = 131071 - max(m, n)
        b = orc.rope(q, m + delta) @ orc.rope(k, n + delta)
        assert abs(a - b) < 1e-9 * (1 + abs(a))


# -------------------------------------------------------------- append ----

def test_append_matches_library_matvec(orc):
    rng = np.random.default_rng(2)
    w, _, dm = _rand_problem(rng)
    p = orc.dims(**dm)
    h = rng.standard_normal((5, dm["d"]))
    rows0 = orc.append_rows(p, h, w["W_DKV"], w["W_KR"], np.zeros(5, np.int32))
    assert np.allclose(rows0[:, : dm["d_c"]], h @ w["W_DKV"].T, rtol=1e-13, atol=1e-13)
    assert np.allclose(rows0[:, dm["d_c"]:], h @ w["W_KR"].T, rtol=1e-13, atol=1e-13)
    pos = np.array([3, 3, 3, 900, 7], np.int32)
    rows = orc.append_rows(p, h, w["W_DKV"], w["W_KR"], pos)
    assert np.allclose(rows[:, : dm["d_c"]], rows0[:, : dm["d_c"]], rtol=0, atol=0)
    kr, kr0 = rows[:, dm["d_c"]:], rows0[:, dm["d_c"]:]
    # rotation keeps norms, and rows at the same position keep their dot products
    assert np.allclose(np.linalg.norm(kr, axis=1), np.linalg.norm(kr0, axis=1), rtol=1e-13)
    assert abs(kr[0] @ kr[1] - kr0[0] @ kr0[1]) < 1e-12
    assert abs(kr[0] @ kr[3] - kr0[0] @ kr0[3]) > 1e-6  # different positions do rotate


# -------------------------------------------------------------- absorb ----

def test_absorb_matches_library_chain(orc):
    rng = np.random.default_rng(3)
    w, _, dm = _rand_problem(rng)
    p = orc.dims(**dm)
    T = 4
    h = rng.standard_normal((T, dm["d"]))
    q, qc = orc.absorb_q(p, h, w["W_DQ"], w["W_UQ"], w["W_QR"], w["W_UK"], np.zeros(T, np.int32),
                         want_qc=True)
    cq = h @ w["W_DQ"].T
    n_h, d_h, d_c, d_r = dm["n_h"], dm["d_h"], dm["d_c"], dm["d_r"]
    for hh in range(n_h):
        WUQ = w["W_UQ"][hh * d_h:(hh + 1) * d_h]
        WUK = w["W_UK"][hh * d_h:(hh + 1) * d_h]
        WQR = w["W_QR"][hh * d_r:(hh + 1) * d_r]
        assert np.allclose(qc[:, hh], cq @ WUQ.T, rtol=1e-12, atol=1e-13)
        # merged matrix (offline absorption W_UK_h^T W_UQ_h) gives the same absorbed query
        merged = WUK.T @ WUQ
        assert np.allclose(q[:, hh, :d_c], cq @ merged.T, rtol=1e-12, atol=1e-13)
        assert np.allclose(q[:, hh, d_c:], cq @ WQR.T, rtol=1e-12, atol=1e-13)


# -------------------------------------------------------------- decode ----

def test_decode_hand_examples(orc):
    ex = json.load(open(os.path.join(GOLDEN, "hand_examples.json")))
    p = orc.dims(d=2, n_h=1, d_h=2, d_c=2, d_cq=2, d_r=2)
    for e in ex["examples"]:
        rows = np.array(e["rows"], np.float64)
        cache = orc.Cache(rows[None])
        q = np.array(e["q"], np.float64).reshape(1, 1, 4)
        o, lse = orc.decode(p, q, cache, np.array([len(rows)], np.int32), 1)
        assert np.allclose(o[0, 0], e["o_lat"], rtol=1e-14, atol=1e-15), e["why"]
        assert abs(lse[0, 0] - e["lse"]) < 1e-14, e["why"]


def test_order_a_equals_order_b(orc):
    # Section 3 of the walk-through: decompress-then-dot (A) and absorb (B)
    # are the same product by associativity; fp64 agreement to 1e-10.
    rng = np.random.default_rng(4)
    for n_q, lens in ((1, (1, 7, 13)), (2, (2, 9, 16))):
        w, seq_lens, dm = _rand_problem(rng, B=3, n_q=n_q, lens=lens)
        p = orc.dims(**dm)
        cache, _ = _build_cache_by_append(orc, p, w, rng, seq_lens)
        c = orc.Cache(cache)
        T = 3 * n_q
        h = rng.standard_normal((T, dm["d"]))
        pos = np.array([seq_lens[t // n_q] - n_q + t % n_q for t in range(T)], np.int32)
        q, qc = orc.absorb_q(p, h, w["W_DQ"], w["W_UQ"], w["W_QR"], w["W_UK"], pos, want_qc=True)
        o_lat, _ = orc.decode(p, q, c, seq_lens, n_q)
        o_b = orc.out_proj(p, o_lat, w["W_UV"]).reshape(T, dm["n_h"], dm["d_h"])
        q_R = q[:, :, dm["d_c"]:]
        o_a = orc.decode_order_a(p, qc, q_R, w["W_UK"], w["W_UV"], c, seq_lens, n_q)
        rel = np.abs(o_a - o_b).max() / np.abs(o_a).max()
        assert rel < 1e-10, rel


def test_decode_special_cases(orc):
    rng = np.random.default_rng(5)
    p = orc.dims(d=8, n_h=2, d_h=4, d_c=8, d_cq=8, d_r=4)
    D = 12
    # L = 1: the output is the single cached latent row, lse its score
    row = rng.standard_normal(D)
    q = rng.standard_normal((1, 2, D))
    o, lse = orc.decode(p, q, orc.Cache(row.reshape(1, 1, D)), np.array([1], np.int32), 1)
    assert np.array_equal(o[0, 0], row[:8]) and np.array_equal(o[0, 1], row[:8])
    assert abs(lse[0, 0] - (q[0, 0] @ row) / math.sqrt(8)) < 1e-14
    # identical rows: any query returns that row
    rows = np.tile(row, (37, 1))
    o, _ = orc.decode(p, q, orc.Cache(rows[None]), np.array([37], np.int32), 1)
    assert np.allclose(o[0], row[:8], rtol=1e-14, atol=1e-14)
    # q = 0: uniform average, lse = log L (softmax weights sum to one)
    rows = rng.standard_normal((23, D))
    o, lse = orc.decode(p, np.zeros((1, 2, D)), orc.Cache(rows[None]), np.array([23], np.int32), 1)
    assert np.allclose(o[0, 0], rows[:, :8].mean(0), rtol=1e-13, atol=1e-14)
    assert abs(lse[0, 1] - math.log(23)) < 1e-14


def test_mla_reduces_to_mha(orc):
    # With d_c = n_h*d_h, W_UK = W_UV = I (per-head identity blocks) and
    # W_QR = W_KR = 0, MLA is standard multi-head attention over K = V = the
    # head's slice of c_KV, scale 1/sqrt(d_h + d_R). Reference: torch SDPA, fp64.
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(6)
    n_h, d_h, d_r, L = 3, 4, 2, 11
    d_c = n_h * d_h
    p = orc.dims(d=d_c, n_h=n_h, d_h=d_h, d_c=d_c, d_cq=d_c, d_r=d_r)
    eye = np.eye(d_c)
    W_UK = eye.copy()
    W_UV = eye.copy()
    ckv = rng.standard_normal((L, d_c))
    rows = np.concatenate([ckv, np.zeros((L, d_r))], 1)
    q_C = rng.standard_normal((1, n_h, d_h))
    q = np.zeros((1, n_h, d_c + d_r))
    for hh in range(n_h):
        q[0, hh, :d_c] = W_UK[hh * d_h:(hh + 1) * d_h].T @ q_C[0, hh]
    o_lat, _ = orc.decode(p, q, orc.Cache(rows[None]), np.array([L], np.int32), 1)
    o = orc.out_proj(p, o_lat, W_UV).reshape(n_h, d_h)
    K = torch.tensor(ckv.reshape(L, n_h, d_h).transpose(1, 0, 2))
    Q = torch.tensor(q_C.reshape(n_h, 1, d_h))
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, K, scale=1 / math.sqrt(d_h + d_r))
    assert np.allclose(o, ref.numpy().reshape(n_h, d_h), rtol=1e-12, atol=1e-13)


def test_order_a_is_sdpa_over_decompressed_heads(orc):
    # Order A (walk-through, section 3: decompress, then dot) is ordinary
    # multi-head attention: per head, keys [W_UK,h c_KV,i ; k_R,i] with the
    # RoPE key shared by all heads, values W_UV,h c_KV,i, query [q_C,h ; q_R,h],
    # scale 1/sqrt(d_h + d_R). Reference: numpy decompression, torch SDPA, fp64.
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(14)
    n_h, d_h, d_c, d_r = 3, 4, 8, 2
    p = orc.dims(d=8, n_h=n_h, d_h=d_h, d_c=d_c, d_cq=8, d_r=d_r)
    lens = (11, 6)
    L = max(lens)
    rows = rng.standard_normal((len(lens), L, d_c + d_r))
    W_UK = rng.standard_normal((n_h * d_h, d_c))
    W_UV = rng.standard_normal((n_h * d_h, d_c))
    q_C = rng.standard_normal((len(lens), n_h, d_h))
    q_R = rng.standard_normal((len(lens), n_h, d_r))
    o = orc.decode_order_a(p, q_C, q_R, W_UK, W_UV, orc.Cache(rows), np.array(lens, np.int32), 1)
    for b, n in enumerate(lens):
        ckv, k_r = rows[b, :n, :d_c], rows[b, :n, d_c:]
        for hh in range(n_h):
            K = np.concatenate([ckv @ W_UK[hh * d_h:(hh + 1) * d_h].T, k_r], 1)
            V = ckv @ W_UV[hh * d_h:(hh + 1) * d_h].T
            Q = np.concatenate([q_C[b, hh], q_R[b, hh]])[None]
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.tensor(Q), torch.tensor(K), torch.tensor(V), scale=1 / math.sqrt(d_h + d_r))
            assert np.allclose(o[b, hh], ref.numpy()[0], rtol=1e-12, atol=1e-13)


def test_split_kv_combine_equals_unsplit(orc):
    rng = np.random.default_rng(7)
    p = orc.dims(d=8, n_h=1, d_h=4, d_c=16, d_cq=8, d_r=4)
    L = 301
    rows = rng.standard_normal((L, 20)) * 2.0
    c = orc.Cache(rows[None])
    q = rng.standard_normal(20) * 3.0
    o_full, lse_full = orc.attend_range(p, q, c, 0, 0, L)
    for cuts in ((0, 150, 301), (0, 1, 2, 64, 300, 301), tuple(range(0, 302, 43)) + (301,)):
        cuts = sorted(set(cuts))
        parts = [orc.attend_range(p, q, c, 0, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
        o, lse = orc.combine(np.stack([x[0] for x in parts]), np.array([x[1] for x in parts]))
        assert np.allclose(o, o_full, rtol=1e-12, atol=1e-13)
        assert abs(lse - lse_full) < 1e-12


def test_paged_slot_mapping_and_equivalence(orc):
    rng = np.random.default_rng(8)
    bs, D = 4, 12
    bt = np.array([[3, 1, 4], [0, 2, 5]], np.int32)
    pool = rng.standard_normal((6, bs, D))
    c = orc.Cache(pool, bt)
    # hand values: slot(b, pos) = block_table[b][pos // bs] * bs + pos % bs
    assert c.slot(0, 5) == 1 * 4 + 1
    assert c.slot(0, 2) == 3 * 4 + 2
    assert c.slot(1, 11) == 5 * 4 + 3
    # the same logical rows laid out contiguously give the same decode
    contig = np.stack([np.concatenate([pool[blk] for blk in bt[b]]) for b in range(2)])
    p = orc.dims(d=8, n_h=2, d_h=4, d_c=8, d_cq=8, d_r=4)
    q = rng.standard_normal((2, 2, D))
    sl = np.array([10, 7], np.int32)
    o1, l1 = orc.decode(p, q, c, sl, 1)
    o2, l2 = orc.decode(p, q, orc.Cache(contig), sl, 1)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_causal_within_step(orc):
    rng = np.random.default_rng(9)
    p = orc.dims(d=8, n_h=2, d_h=4, d_c=8, d_cq=8, d_r=4)
    rows = rng.standard_normal((1, 9, 12))
    q = rng.standard_normal((2, 2, 12))
    sl = np.array([9], np.int32)
    o1, _ = orc.decode(p, q, orc.Cache(rows), sl, 2)
    rows2 = rows.copy()
    rows2[0, 8] += 5.0        # the second new token (position 8)
    o2, _ = orc.decode(p, q, orc.Cache(rows2), sl, 2)
    assert np.array_equal(o1[0], o2[0])          # query 0 sits at position 7
    assert not np.allclose(o1[1], o2[1])         # query 1 sees position 8


def test_rope_shift_invariance_end_to_end(orc):
    # Relative position: moving every cached key and the query by the same
    # offset leaves the decode result unchanged.
    rng = np.random.default_rng(10)
    w, seq_lens, dm = _rand_problem(rng, B=1, lens=(12,))
    p = orc.dims(**dm)
    c0, hs = _build_cache_by_append(orc, p, w, rng, seq_lens, shift=0)
    c1, _ = _build_cache_by_append(orc, p, w, rng, seq_lens, shift=131060 - 11, hs=hs)
    hq = rng.standard_normal((1, dm["d"]))
    q0 = orc.absorb_q(p, hq, w["W_DQ"], w["W_UQ"], w["W_QR"], w["W_UK"], np.array([11], np.int32))
    q1 = orc.absorb_q(p, hq, w["W_DQ"], w["W_UQ"], w["W_QR"], w["W_UK"], np.array([131060], np.int32))
    o0, _ = orc.decode(p, q0, orc.Cache(c0), seq_lens, 1)
    o1, _ = orc.decode(p, q1, orc.Cache(c1), seq_lens, 1)
    assert np.allclose(o0, o1, rtol=1e-9, atol=1e-11)


def test_out_proj_matches_library(orc):
    rng = np.random.default_rng(11)
    p = orc.dims(d=8, n_h=3, d_h=4, d_c=6, d_cq=8, d_r=2)
    o_lat = rng.standard_normal((5, 3, 6))
    W_UV = rng.standard_normal((12, 6))
    o = orc.out_proj(p, o_lat, W_UV)
    ref = np.einsum("hij,thj->thi", W_UV.reshape(3, 4, 6), o_lat).reshape(5, 12)
    assert np.allclose(o, ref, rtol=1e-13, atol=1e-14)


# ------------------------------------ output projection W_O (next row) ----

def test_o_proj_matches_library(orc):
    # walk-through step 5: the concatenated head outputs times W_O (d x n_h d_h)
    rng = np.random.default_rng(12)
    W_O = rng.standard_normal((7, 12))
    o = rng.standard_normal((5, 12))
    assert np.allclose(orc.o_proj(W_O, o), o @ W_O.T, rtol=1e-13, atol=1e-14)


def test_absorbed_w_o_matches_library_and_the_two_stage_readout(orc):
    # W_UV absorbed into W_O: W_OV[r][h d_c + j] = sum_i W_O[r][h d_h + i] W_UV[h d_h + i][j]
    rng = np.random.default_rng(13)
    n_h, d_h, d_c, d = 3, 4, 6, 7
    p = orc.dims(d=d, n_h=n_h, d_h=d_h, d_c=d_c, d_cq=8, d_r=2)
    W_O = rng.standard_normal((d, n_h * d_h))
    W_UV = rng.standard_normal((n_h * d_h, d_c))
    W_OV = orc.absorb_wo(p, W_O, W_UV)
    ref = np.einsum("rhi,hij->rhj", W_O.reshape(d, n_h, d_h), W_UV.reshape(n_h, d_h, d_c)).reshape(d, n_h * d_c)
    assert np.allclose(W_OV, ref, rtol=1e-13, atol=1e-14)
    # reading out in latent space with W_OV equals decompressing with W_UV, then W_O
    o_lat = rng.standard_normal((5, n_h, d_c))
    one_stage = orc.o_proj(W_OV, o_lat.reshape(5, n_h * d_c))
    two_stage = orc.o_proj(W_O, orc.out_proj(p, o_lat, W_UV))
    assert np.allclose(one_stage, two_stage, rtol=1e-12, atol=1e-13)


def test_merged_absorption_matches_the_two_stage_query(orc):
    # the merged matrix W_UK_h^T W_UQ_h (walk-through section 3, order B): applied to c_Q it
    # gives the oracle's own two-stage q_lat (W_UQ, then W_UK^T), which the library-chain and
    # order-A pins fix independently; and it is the per-head product of the library
    rng = np.random.default_rng(14)
    w, _, dm = _rand_problem(rng)
    p = orc.dims(**dm)
    n_h, d_h, d_c, d_cq = dm["n_h"], dm["d_h"], dm["d_c"], dm["d_cq"]
    W_UQK = orc.absorb_merge(p, w["W_UQ"], w["W_UK"])
    assert W_UQK.shape == (n_h * d_c, d_cq)
    T = 3
    h = rng.standard_normal((T, dm["d"]))
    q = orc.absorb_q(p, h, w["W_DQ"], w["W_UQ"], w["W_QR"], w["W_UK"], np.arange(T, dtype=np.int32))
    cq = h @ w["W_DQ"].T
    for hh in range(n_h):
        assert np.allclose(cq @ W_UQK[hh * d_c:(hh + 1) * d_c].T, q[:, hh, :d_c], rtol=1e-11, atol=1e-12)
    ref = np.einsum("hij,hic->hjc", w["W_UK"].reshape(n_h, d_h, d_c), w["W_UQ"].reshape(n_h, d_h, d_cq))
    assert np.allclose(W_UQK, ref.reshape(n_h * d_c, d_cq), rtol=1e-13, atol=1e-14)


def test_bf16_cache_read_is_exact(orc):
    # the oracle reads bf16 storage as the exact real value of those bits
    vals = np.array([1.0, -2.5, 3.140625, 1e-3, 65280.0], np.float32)
    bits = synth.bf16_bits(vals)
    back = synth.bf16_to_f32(bits)
    assert back[0] == 1.0 and back[1] == -2.5 and back[2] == 3.140625 and back[4] == 65280.0
    p = orc.dims(d=2, n_h=1, d_h=2, d_c=4, d_cq=2, d_r=1)
    rows = bits[None, None, :]
    o, _ = orc.decode(p, np.zeros((1, 1, 5)), orc.Cache(rows), np.array([1], np.int32), 1)
    assert np.array_equal(o[0, 0], back[:4].astype(np.float64))


# ----------------------------------------------- cache size (page numbers) --

def test_cache_size_claims_from_pages():
    g = json.load(open(os.path.join(GOLDEN, "page_dims.json")))
    v2 = g["deepseek_v2"]
    w = synth.WORKLOADS["v2_b16_4k"]
    for k in ("d", "n_h", "d_h", "d_c", "d_cq", "d_r"):
        assert getattr(w, k) == v2[k]
    assert w.d_h + w.d_r == v2["score_dim"]
    assert w.n_h * w.d_h == v2["concat_dim"]
    mla_per_token = w.d_c + w.d_r
    mha_per_token = 2 * w.n_h * w.d_h
    assert (mla_per_token, mha_per_token) == (576, 32768)
    ex = g["compression_example"]
    ratio = ex["d_c"] / (2 * ex["n_h"] * ex["d_h"])
    assert ratio == ex["ratio"] and 100 * (1 - ratio) == ex["reduction_pct"]


def test_synth_is_seeded_and_shaped():
    w = synth.shrink(synth.WORKLOADS["v2_b64_paged"], B=3, L_lo=5, L_hi=130, d=64, d_cq=32)
    a, b = synth.generate(w), synth.generate(w)
    assert np.array_equal(a.cache, b.cache) and np.array_equal(a.h, b.h)
    assert a.cache.shape[1:] == (64, 576) and a.block_table.shape[0] == 3
    assert np.all(a.positions == a.seq_lens - 1)
    # every block id appears once
    ids = np.concatenate([a.block_table[i, : (a.seq_lens[i] + 63) // 64] for i in range(3)])
    assert len(np.unique(ids)) == len(ids) == a.cache.shape[0]
