"""fp64 CPU oracle for absorbed-form MLA decode — TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
arm may import this package. The CUDA library never calls it.

This module is argument marshalling for the plain-C oracle in mla_oracle.c
(numpy arrays -> float64 pointers); all arithmetic is in that file. Sources
are cited there: the MLA walk-through (h.sjds.net, section 1 steps 1-5 and
section 3 orders A/B), the DeepSeek-V2 MLA explainer (modelers.csdn.net,
equations 9-13 and the absorption remark) and the RoPE tutorial
(xianlaiwan.cn).
"""
import ctypes as C

import numpy as np

from . import build as _build

_lib = None


class OrcDims(C.Structure):
    _fields_ = [("d", C.c_int32), ("n_h", C.c_int32), ("d_h", C.c_int32), ("d_c", C.c_int32),
                ("d_cq", C.c_int32), ("d_r", C.c_int32), ("rope_base", C.c_double),
                ("scale", C.c_double)]


class OrcCache(C.Structure):
    _fields_ = [("data", C.c_void_p), ("dtype", C.c_int32), ("paged", C.c_int32),
                ("block_size", C.c_int32), ("max_blocks_per_seq", C.c_int32),
                ("block_table", C.c_void_p), ("max_len", C.c_int64)]


_P = C.c_void_p


def bind(L):
    """Declare the C signatures on a loaded liboracle (argument marshalling)."""
    L.orc_rope.argtypes = [_P, C.c_int, C.c_double, C.c_double]
    L.orc_slot.argtypes = [C.POINTER(OrcCache), C.c_int32, C.c_int64]
    L.orc_slot.restype = C.c_int64
    L.orc_append.argtypes = [C.POINTER(OrcDims), _P, _P, _P, _P, C.c_int, _P]
    L.orc_absorb_q.argtypes = [C.POINTER(OrcDims), _P, _P, _P, _P, _P, _P, C.c_int, _P, _P]
    L.orc_decode.argtypes = [C.POINTER(OrcDims), _P, C.POINTER(OrcCache), _P, C.c_int, C.c_int,
                             _P, _P, _P, C.c_int]
    L.orc_decode.restype = C.c_int
    L.orc_attend_range.argtypes = [C.POINTER(OrcDims), _P, C.POINTER(OrcCache), C.c_int32,
                                   C.c_int64, C.c_int64, _P, _P]
    L.orc_combine.argtypes = [C.c_int, C.c_int, _P, _P, _P, _P]
    L.orc_out_proj.argtypes = [C.POINTER(OrcDims), _P, _P, C.c_int, _P]
    L.orc_decode_order_a.argtypes = [C.POINTER(OrcDims), _P, _P, _P, _P, C.POINTER(OrcCache),
                                     _P, C.c_int, C.c_int, _P, _P, C.c_int]
    L.orc_decode_order_a.restype = C.c_int
    L.orc_o_proj.argtypes = [_P, C.c_int, C.c_int, _P, C.c_int, _P]
    L.orc_absorb_wo.argtypes = [C.POINTER(OrcDims), _P, _P, _P]
    L.orc_absorb_merge.argtypes = [C.POINTER(OrcDims), _P, _P, _P]
    L.orc_set_threads.argtypes = [C.c_int]
    L.orc_max_threads.restype = C.c_int
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = bind(C.CDLL(_build.build()))
    return _lib


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def max_threads() -> int:
    return int(lib().orc_max_threads())


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def dims(d, n_h, d_h, d_c, d_cq, d_r, rope_base=10000.0, scale=0.0) -> OrcDims:
    return OrcDims(int(d), int(n_h), int(d_h), int(d_c), int(d_cq), int(d_r), float(rope_base),
                   float(scale))


class Cache:
    """A cache held in its storage format for the oracle.

    data: numpy array whose last dim is d_c + d_r. dtype uint16 = bf16 bit
    patterns, float32 or float64. Contiguous: [num_seqs][max_len][D].
    Paged: [num_blocks][block_size][D] with block_table [num_seqs][max_blocks].
    """

    def __init__(self, data, block_table=None):
        self.data = np.ascontiguousarray(data)
        if self.data.dtype == np.uint16:
            code = 0
        elif self.data.dtype == np.float32:
            code = 1
        elif self.data.dtype == np.float64:
            code = 2
        else:
            raise TypeError(f"unsupported cache dtype {self.data.dtype}")
        self.block_table = None if block_table is None else _i32(block_table)
        if self.block_table is None:
            self.c = OrcCache(self.data.ctypes.data, code, 0, 0, 0, None, self.data.shape[1])
        else:
            self.c = OrcCache(self.data.ctypes.data, code, 1, self.data.shape[1],
                              self.block_table.shape[1], self.block_table.ctypes.data, 0)

    def slot(self, b: int, pos: int) -> int:
        return int(lib().orc_slot(C.byref(self.c), int(b), int(pos)))


def rope(x, pos, base=10000.0):
    x = _f64(x).copy()
    lib().orc_rope(_ptr(x), x.shape[-1], float(pos), float(base))
    return x


def append_rows(p: OrcDims, h, W_DKV, W_KR, positions):
    h, W_DKV, W_KR, pos = _f64(h), _f64(W_DKV), _f64(W_KR), _i32(positions)
    T = h.shape[0]
    rows = np.zeros((T, p.d_c + p.d_r), np.float64)
    lib().orc_append(C.byref(p), _ptr(h), _ptr(W_DKV), _ptr(W_KR), _ptr(pos), T, _ptr(rows))
    return rows


def absorb_q(p: OrcDims, h, W_DQ, W_UQ, W_QR, W_UK, positions, want_qc=False):
    h, W_DQ, W_UQ, W_QR, W_UK = map(_f64, (h, W_DQ, W_UQ, W_QR, W_UK))
    pos = _i32(positions)
    T = h.shape[0]
    q = np.zeros((T, p.n_h, p.d_c + p.d_r), np.float64)
    qc = np.zeros((T, p.n_h, p.d_h), np.float64) if want_qc else None
    lib().orc_absorb_q(C.byref(p), _ptr(h), _ptr(W_DQ), _ptr(W_UQ), _ptr(W_QR), _ptr(W_UK),
                       _ptr(pos), T, _ptr(q), _ptr(qc))
    return (q, qc) if want_qc else q


def decode(p: OrcDims, q, cache: Cache, seq_lens, n_q, pairs=None):
    """Order B. Returns (o_lat, lse): [T][n_h][d_c], [T][n_h] or, with pairs
    (array of (t, h)), [n_pairs][d_c], [n_pairs]."""
    q = _f64(q)
    sl = _i32(seq_lens)
    B = sl.shape[0]
    if pairs is None:
        o = np.zeros((B * n_q, p.n_h, p.d_c), np.float64)
        lse = np.zeros((B * n_q, p.n_h), np.float64)
        pr, n_pairs = None, 0
    else:
        pr = _i32(pairs).reshape(-1, 2)
        n_pairs = pr.shape[0]
        o = np.zeros((n_pairs, p.d_c), np.float64)
        lse = np.zeros((n_pairs,), np.float64)
    rc = lib().orc_decode(C.byref(p), _ptr(q), C.byref(cache.c), _ptr(sl), B, int(n_q), _ptr(o),
                          _ptr(lse), _ptr(pr), n_pairs)
    if rc != 0:
        raise ValueError("oracle decode: a sequence is shorter than n_q")
    return o, lse


def attend_range(p: OrcDims, q_row, cache: Cache, b, start, end):
    q_row = _f64(q_row)
    o = np.zeros((p.d_c,), np.float64)
    lse = np.zeros((1,), np.float64)
    lib().orc_attend_range(C.byref(p), _ptr(q_row), C.byref(cache.c), int(b), int(start), int(end),
                           _ptr(o), _ptr(lse))
    return o, float(lse[0])


def combine(o_parts, lse_parts):
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    S, d_c = o_parts.shape
    o = np.zeros((d_c,), np.float64)
    lse = np.zeros((1,), np.float64)
    lib().orc_combine(S, d_c, _ptr(o_parts), _ptr(lse_parts), _ptr(o), _ptr(lse))
    return o, float(lse[0])


def out_proj(p: OrcDims, o_lat, W_UV):
    o_lat, W_UV = _f64(o_lat), _f64(W_UV)
    T = o_lat.shape[0]
    o = np.zeros((T, p.n_h * p.d_h), np.float64)
    lib().orc_out_proj(C.byref(p), _ptr(o_lat), _ptr(W_UV), T, _ptr(o))
    return o


def o_proj(W, x):
    """y[t] = W x[t] (walk-through step 5 with W = W_O and x = the concatenated
    head outputs; or W = W_OV from absorb_wo and x = o_lat flattened)."""
    W = _f64(W)
    x = _f64(x).reshape(-1, W.shape[1])
    y = np.empty((x.shape[0], W.shape[0]))
    lib().orc_o_proj(_ptr(W), W.shape[0], W.shape[1], _ptr(x), x.shape[0], _ptr(y))
    return y


def absorb_wo(p: OrcDims, W_O, W_UV):
    """W_OV (d x n_h*d_c): W_UV absorbed into W_O."""
    W_O, W_UV = _f64(W_O), _f64(W_UV)
    W_OV = np.empty((p.d, p.n_h * p.d_c))
    lib().orc_absorb_wo(C.byref(p), _ptr(W_O), _ptr(W_UV), _ptr(W_OV))
    return W_OV


def absorb_merge(p: OrcDims, W_UQ, W_UK):
    """W_UQK (n_h*d_c x d_cq): the merged absorption matrix W_UK_h^T W_UQ_h per head."""
    W_UQ, W_UK = _f64(W_UQ), _f64(W_UK)
    W_UQK = np.empty((p.n_h * p.d_c, p.d_cq))
    lib().orc_absorb_merge(C.byref(p), _ptr(W_UQ), _ptr(W_UK), _ptr(W_UQK))
    return W_UQK


def decode_order_a(p: OrcDims, q_C, q_R, W_UK, W_UV, cache: Cache, seq_lens, n_q, pairs=None):
    """Order A (decompress per head, then ordinary attention). Returns o per
    head: [T][n_h][d_h] or [n_pairs][d_h]."""
    q_C, q_R, W_UK, W_UV = map(_f64, (q_C, q_R, W_UK, W_UV))
    sl = _i32(seq_lens)
    B = sl.shape[0]
    if pairs is None:
        o = np.zeros((B * n_q, p.n_h, p.d_h), np.float64)
        pr, n_pairs = None, 0
    else:
        pr = _i32(pairs).reshape(-1, 2)
        n_pairs = pr.shape[0]
        o = np.zeros((n_pairs, p.d_h), np.float64)
    rc = lib().orc_decode_order_a(C.byref(p), _ptr(q_C), _ptr(q_R), _ptr(W_UK), _ptr(W_UV),
                                  C.byref(cache.c), _ptr(sl), B, int(n_q), _ptr(o), _ptr(pr),
                                  n_pairs)
    if rc != 0:
        raise ValueError("oracle order A: a sequence is shorter than n_q")
    return o


def step(p: OrcDims, w, h, positions, seq_idx, cache_rows_before: Cache, seq_lens, n_q):
    """Whole hot path in fp64: append the new rows into a float64 copy of the
    cache, absorb the query, decode (order B) and up-project with W_UV.

    w: dict of float64-convertible weights; returns dict with rows, q, o_lat,
    lse, o and the float64 cache after the append.
    """
    rows = append_rows(p, h, w["W_DKV"], w["W_KR"], positions)
    data = cache_rows_before.data
    if data.dtype == np.uint16:
        u = data.astype(np.uint32) << 16
        data64 = u.view(np.float32).astype(np.float64)
    else:
        data64 = data.astype(np.float64)
    c64 = Cache(data64, cache_rows_before.block_table)
    flat = c64.data.reshape(-1, p.d_c + p.d_r)
    for t in range(rows.shape[0]):
        flat[c64.slot(int(seq_idx[t]), int(positions[t]))] = rows[t]
    q = absorb_q(p, h, w["W_DQ"], w["W_UQ"], w["W_QR"], w["W_UK"], positions)
    o_lat, lse = decode(p, q, c64, seq_lens, n_q)
    o = out_proj(p, o_lat, w["W_UV"])
    return {"rows": rows, "q": q, "o_lat": o_lat, "lse": lse, "o": o, "cache": c64}


__all__ = ["dims", "Cache", "rope", "append_rows", "absorb_q", "decode", "attend_range",
           "combine", "out_proj", "decode_order_a", "step", "set_threads", "max_threads", "o_proj",
           "absorb_wo", "absorb_merge"]

