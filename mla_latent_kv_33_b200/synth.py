"""Seeded synthetic inputs for the MLA decode hot path.

This module only draws random numbers and packs them into storage formats
(bf16 bit patterns, fp32). It holds none of the method's arithmetic (no
projection, no RoPE, no softmax), so both the fp64 oracle and the CUDA path
can consume its output.

Recipe (one ``numpy.random.Generator(PCG64(seed))`` per workload):
  weights in the order W_DKV, W_KR, W_DQ, W_UQ, W_QR, W_UK, W_UV, each
  N(0, 1/fan_in) with fan_in the input width (d for W_DKV/W_KR/W_DQ, d_c' for
  W_UQ/W_QR, d_c for W_UK/W_UV), rounded once to the storage dtype; then the
  new tokens' hidden states h ~ N(0, 1); then the sequence lengths; then the
  paged-pool block permutation; then the prefilled cache rows ~ N(0, 1).

Prefilled rows stand in for earlier appends: each coordinate of W_DKV h is
N(0, 1) under this weight scaling, and a RoPE rotation of an isotropic
Gaussian pair is again isotropic Gaussian, so N(0, 1) rows have the same
distribution as appended rows without running the method here. Slots that
hold no token (past the sequence end inside its last block, and the slots
this step's append will write) are filled with a NaN canary so that any read
of them would show up in the outputs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

BF16_NAN = np.uint16(0x7FC1)     # quiet NaN canary (bf16 bits)
F32_NAN_BITS = np.uint32(0x7FC00001)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Workload:
    name: str
    index: int                 # position in the workload table; seed = 1000 + index
    d: int
    n_h: int
    d_h: int
    d_c: int
    d_cq: int
    d_r: int
    B: int
    n_q: int
    lens: str                  # "fixed" | "uniform" | "lognormal"
    L: int = 0                 # fixed length
    L_lo: int = 0
    L_hi: int = 0
    median: float = 0.0
    sigma: float = 0.0
    paged: bool = False
    block_size: int = 64
    dtype: str = "bf16"        # storage dtype: "bf16" | "fp32"
    prefill: str = "random"    # "random" rows or "append" (run the append on extra tokens)
    rope_base: float = 10000.0
    note: str = ""

    @property
    def D(self) -> int:
        return self.d_c + self.d_r

    @property
    def T(self) -> int:
        return self.B * self.n_q


V2 = dict(d=5120, n_h=128, d_h=128, d_c=512, d_cq=1536, d_r=64)
V3 = dict(d=7168, n_h=128, d_h=128, d_c=512, d_cq=1536, d_r=64)

WORKLOADS = {
    "tiny_fp32": Workload(
        "tiny_fp32", 0, d=256, n_h=4, d_h=32, d_c=64, d_cq=96, d_r=16, B=1, n_q=1, lens="fixed",
        L=65, dtype="fp32", prefill="append",
        note="tiny MLA single decode step, fp32; 64 cached tokens + 1 query at position 64"),
    "v2_b16_4k": Workload(
        "v2_b16_4k", 1, **V2, B=16, n_q=1, lens="fixed", L=4096,
        note="DeepSeek-V2 layer decode, batch 16, context 4096, contiguous latent cache"),
    "v2_b64_paged": Workload(
        "v2_b64_paged", 2, **V2, B=64, n_q=1, lens="uniform", L_lo=1024, L_hi=8192, paged=True,
        note="DeepSeek-V2 dims, batch 64, seq_lens ~ U[1024, 8192], paged cache (block 64)"),
    "v2_b4_128k": Workload(
        "v2_b4_128k", 3, **V2, B=4, n_q=1, lens="fixed", L=131072, paged=True,
        note="DeepSeek-V2 dims, batch 4, context 131072, paged cache, split-KV"),
    "v3_b128_nq2": Workload(
        "v3_b128_nq2", 4, **V3, B=128, n_q=2, lens="lognormal", median=4096.0, sigma=0.5,
        L_lo=256, L_hi=32768, paged=True,
        note="DeepSeek-V3 dims, batch 128, lognormal seq_lens (median 4096, sigma 0.5, "
             "clipped 256..32768), 2 query tokens per sequence"),
    "v2_prefill_c512": Workload(
        "v2_prefill_c512", 5, **V2, B=4, n_q=512, lens="fixed", L=4096, paged=True,
        note="DeepSeek-V2 dims, chunked prefill: 4 sequences, a chunk of 512 new tokens each at positions "
             "3584..4095 (causal within the chunk), paged cache (block 64); the order-A (training form) workload"),
}


def shrink(w: Workload, **kw) -> Workload:
    """Same recipe at other sizes (parity-test cases)."""
    return replace(w, **kw)


@dataclass
class Inputs:
    w: Workload
    weights: dict                     # name -> float32 array holding storage-exact values
    weights_bits: dict                # name -> uint16 bf16 bits (bf16 workloads only)
    h: np.ndarray                     # [T][d] float32, storage-exact values
    h_bits: np.ndarray | None
    seq_lens: np.ndarray              # [B] int32, after this step's append
    positions: np.ndarray             # [T] int32
    seq_idx: np.ndarray               # [T] int32
    cache: np.ndarray                 # storage array; uint16 bits (bf16) or float32
    block_table: np.ndarray | None    # [B][max_blocks] int32
    prefill_h: np.ndarray | None = None    # tokens appended before the step ("append" prefill)
    prefill_pos: np.ndarray | None = None
    prefill_seq: np.ndarray | None = None
    extra: dict = field(default_factory=dict)


def _round_store(x: np.ndarray, dtype: str):
    """Return (float32 values exactly representable in storage, bits or None)."""
    x = np.asarray(x, dtype=np.float32)
    if dtype == "bf16":
        bits = bf16_bits(x)
        return bf16_to_f32(bits), bits
    return x.copy(), None


def _lengths(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.lens == "fixed":
        L = np.full((w.B,), w.L, dtype=np.int64)
    elif w.lens == "uniform":
        L = rng.integers(w.L_lo, w.L_hi + 1, size=w.B, dtype=np.int64)
    elif w.lens == "lognormal":
        z = rng.standard_normal(w.B)
        L = np.clip(np.rint(np.exp(math.log(w.median) + w.sigma * z)), w.L_lo, w.L_hi).astype(np.int64)
    else:
        raise ValueError(w.lens)
    L = np.maximum(L, w.n_q)
    return L.astype(np.int32)


def generate(w: Workload, seed: int | None = None, cache_headroom_blocks: int = 0) -> Inputs:
    rng = np.random.Generator(np.random.PCG64(1000 + w.index if seed is None else seed))
    shapes = {
        "W_DKV": (w.d_c, w.d), "W_KR": (w.d_r, w.d), "W_DQ": (w.d_cq, w.d),
        "W_UQ": (w.n_h * w.d_h, w.d_cq), "W_QR": (w.n_h * w.d_r, w.d_cq),
        "W_UK": (w.n_h * w.d_h, w.d_c), "W_UV": (w.n_h * w.d_h, w.d_c),
    }
    weights, weights_bits = {}, {}
    for name, shp in shapes.items():
        x = rng.standard_normal(shp, dtype=np.float32) * np.float32(1.0 / math.sqrt(shp[1]))
        weights[name], bits = _round_store(x, w.dtype)
        if bits is not None:
            weights_bits[name] = bits
    h, h_bits = _round_store(rng.standard_normal((w.T, w.d), dtype=np.float32), w.dtype)
    seq_lens = _lengths(w, rng)

    B, n_q, D = w.B, w.n_q, w.D
    positions = np.empty((w.T,), np.int32)
    seq_idx = np.empty((w.T,), np.int32)
    for b in range(B):
        for j in range(n_q):
            positions[b * n_q + j] = seq_lens[b] - n_q + j
            seq_idx[b * n_q + j] = b
    max_len = int(seq_lens.max())

    block_table = None
    if w.paged:
        bs = w.block_size
        nblk = (seq_lens.astype(np.int64) + bs - 1) // bs
        total = int(nblk.sum()) + cache_headroom_blocks
        perm = rng.permutation(total).astype(np.int32)
        max_blocks = int(nblk.max())
        block_table = np.zeros((B, max_blocks), np.int32)
        off = 0
        for b in range(B):
            block_table[b, : nblk[b]] = perm[off: off + nblk[b]]
            off += int(nblk[b])
        rows_shape = (total, bs, D)
    else:
        rows_shape = (B, max_len, D)

    nrows = int(np.prod(rows_shape[:2]))
    if w.dtype == "bf16":
        cache = np.full((nrows, D), BF16_NAN, np.uint16)
    else:
        cache = np.full((nrows, D), F32_NAN_BITS, np.uint32).view(np.float32)

    # logical -> physical row for every cached position that holds a token
    def phys(b, pos):
        if w.paged:
            return block_table[b, pos // w.block_size].astype(np.int64) * w.block_size + pos % w.block_size
        return np.int64(b) * max_len + pos

    prefill_h = prefill_pos = prefill_seq = None
    if w.prefill == "random":
        for b in range(B):
            n = int(seq_lens[b]) - n_q
            if n <= 0:
                continue
            vals = rng.standard_normal((n, D), dtype=np.float32)
            stored, bits = _round_store(vals, w.dtype)
            pos = np.arange(n, dtype=np.int64)
            rows = phys(b, pos)
            cache[rows] = bits if bits is not None else stored
    elif w.prefill == "append":
        n_pre = int((seq_lens - n_q).sum())
        prefill_h, _ = _round_store(rng.standard_normal((n_pre, w.d), dtype=np.float32), w.dtype)
        prefill_pos = np.concatenate([np.arange(int(seq_lens[b]) - n_q, dtype=np.int32) for b in range(B)])
        prefill_seq = np.concatenate([np.full((int(seq_lens[b]) - n_q,), b, np.int32) for b in range(B)])
    else:
        raise ValueError(w.prefill)

    cache = cache.reshape(rows_shape)
    return Inputs(w, weights, weights_bits, h, h_bits, seq_lens, positions, seq_idx, cache,
                  block_table, prefill_h, prefill_pos, prefill_seq)


def algorithmic_work(w: Workload, seq_lens: np.ndarray) -> dict:
    """Bytes of latent cache read and tensor flops the decode must do."""
    L = seq_lens.astype(np.int64)
    # query token j of sequence b sees L_b - n_q + 1 + j cached rows
    vis = sum(int(L[b]) - w.n_q + 1 + j for b in range(w.B) for j in range(w.n_q))
    uniq = int(L.sum())
    elem = 2 if w.dtype == "bf16" else 4
    return {
        "cache_bytes": uniq * w.D * elem,
        "flops": vis * w.n_h * 2 * (w.D + w.d_c),
        "tokens_attended": vis,
    }


@dataclass
class DecodeInputs:
    w: Workload
    q: np.ndarray                     # [T][n_h][D] float32 storage-exact
    q_bits: np.ndarray | None
    seq_lens: np.ndarray
    cache: np.ndarray
    block_table: np.ndarray | None


def generate_decode(w: Workload, seed: int, seq_lens=None, q_scale: float = 0.5) -> DecodeInputs:
    """Inputs of the decode step alone: absorbed queries drawn directly
    (q_lat ~ N(0, q_scale^2), q_R ~ N(0, 1): the spread the absorb step gives
    under the weight scaling above) and a cache of N(0, 1) rows, NaN canaries
    in unused slots. seq_lens (optional) overrides the workload's length recipe."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if seq_lens is None:
        seq_lens = _lengths(w, rng)
    seq_lens = np.asarray(seq_lens, np.int32)
    w = replace(w, B=len(seq_lens))
    qv = rng.standard_normal((w.T, w.n_h, w.D), dtype=np.float32)
    qv[:, :, : w.d_c] *= np.float32(q_scale)
    q, q_bits = _round_store(qv, w.dtype)
    B, D = w.B, w.D
    block_table = None
    if w.paged:
        bs = w.block_size
        nblk = (seq_lens.astype(np.int64) + bs - 1) // bs
        total = int(nblk.sum())
        perm = rng.permutation(total).astype(np.int32)
        block_table = np.zeros((B, int(nblk.max())), np.int32)
        off = 0
        for b in range(B):
            block_table[b, : nblk[b]] = perm[off: off + nblk[b]]
            off += int(nblk[b])
        shape = (total, bs, D)
    else:
        shape = (B, int(seq_lens.max()), D)
    nrows = shape[0] * shape[1]
    if w.dtype == "bf16":
        cache = np.full((nrows, D), BF16_NAN, np.uint16)
    else:
        cache = np.full((nrows, D), F32_NAN_BITS, np.uint32).view(np.float32)
    for b in range(B):
        n = int(seq_lens[b])
        vals = rng.standard_normal((n, D), dtype=np.float32)
        stored, bits = _round_store(vals, w.dtype)
        pos = np.arange(n, dtype=np.int64)
        if w.paged:
            rows = block_table[b, pos // w.block_size].astype(np.int64) * w.block_size + pos % w.block_size
        else:
            rows = np.int64(b) * shape[1] + pos
        cache[rows] = bits if bits is not None else stored
    return DecodeInputs(w, q, q_bits, seq_lens, cache.reshape(shape), block_table)
