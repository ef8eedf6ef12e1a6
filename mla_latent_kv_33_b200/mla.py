"""ctypes binding of libmla.so (include/mla.h): argument marshalling only.

Every function here forwards to the C entry point of the same name with
device pointers taken from torch tensors (torch is used for device memory and
streams). No step of the computation runs in Python, and there is no fallback:
if the library is missing this module raises on import.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m mla_latent_kv_33_b200.build`")

_lib = C.CDLL(LIB_PATH)

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_WORKSPACE, MLA_ERR_CUDA, MLA_ERR_TIMEOUT, \
    MLA_ERR_DEVICE_DATA = range(7)
MLA_BF16, MLA_FP32 = 0, 1
OP_APPEND, OP_ABSORB, OP_DECODE, OP_OUT_PROJ, OP_O_PROJ, OP_O_PROJ_LATENT, OP_ABSORB_MERGED, OP_FRONT_END, \
    OP_ABSORB_WO, OP_QUERY_HEADS, OP_ATTEND_A = range(11)


class Dims(C.Structure):
    _fields_ = [("d", C.c_int32), ("n_h", C.c_int32), ("d_h", C.c_int32), ("d_c", C.c_int32),
                ("d_cq", C.c_int32), ("d_r", C.c_int32), ("rope_base", C.c_double),
                ("softmax_scale", C.c_float), ("dtype", C.c_int32)]


class CacheDesc(C.Structure):
    _fields_ = [("data", C.c_void_p), ("paged", C.c_int32), ("block_size", C.c_int32),
                ("block_table", C.c_void_p), ("max_blocks_per_seq", C.c_int32),
                ("num_seqs", C.c_int32), ("max_len", C.c_int64), ("num_blocks", C.c_int64)]


_P, _S = C.c_void_p, C.c_size_t
_lib.mla_cache_append.argtypes = [C.POINTER(Dims), _P, _P, _P, _P, _P, C.c_int32, C.POINTER(CacheDesc),
                                  _P, _S, _P]
_lib.mla_absorb_q.argtypes = [C.POINTER(Dims), _P, _P, _P, _P, _P, _P, C.c_int32, _P, _P, _S, _P]
_lib.mla_decode.argtypes = [C.POINTER(Dims), _P, C.POINTER(CacheDesc), _P, C.c_int32, C.c_int32, _P, _P,
                            C.c_int32, _P, _S, _P]
_lib.mla_out_proj.argtypes = [C.POINTER(Dims), _P, _P, C.c_int32, _P, _P, _S, _P]
_lib.mla_o_proj.argtypes = [C.POINTER(Dims), _P, _P, C.c_int32, _P, _P, _S, _P]
_lib.mla_decode_noalloc.argtypes = [C.POINTER(Dims), _P, C.POINTER(CacheDesc), _P, C.c_int32, C.c_int32, _P, _P, _P]
_lib.mla_absorb_wo.argtypes = [C.POINTER(Dims), _P, _P, _P, _P]
_lib.mla_o_proj_latent.argtypes = [C.POINTER(Dims), _P, _P, C.c_int32, _P, _P, _S, _P]
_lib.mla_absorb_merge.argtypes = [C.POINTER(Dims), _P, _P, _P, _P]
_lib.mla_absorb_q_merged.argtypes = [C.POINTER(Dims), _P, _P, _P, _P, _P, C.c_int32, _P, _P, _S, _P]
_lib.mla_front_end.argtypes = [C.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P, _P, _P, C.c_int32,
                               C.POINTER(CacheDesc), _P, _P, _S, _P]
_lib.mla_selftest_timeout.argtypes = [C.c_uint64, _P, _S, _P]
_lib.mla_query_heads.argtypes = [C.POINTER(Dims), _P, _P, _P, _P, _P, C.c_int32, _P, _P, _S, _P]
_lib.mla_attend_order_a.argtypes = [C.POINTER(Dims), _P, _P, _P, C.POINTER(CacheDesc), _P, C.c_int32, C.c_int32, _P,
                                    _P, _S, _P]
_lib.mla_workspace_size.argtypes = [C.POINTER(Dims), C.c_int32, C.c_int32, C.c_int32, C.c_int64, C.c_int32]
_lib.mla_workspace_size.restype = C.c_size_t
_lib.mla_get_device_error.argtypes = [_P]
_lib.mla_status_string.argtypes = [C.c_int]
_lib.mla_status_string.restype = C.c_char_p
_lib.mla_last_error_message.restype = C.c_char_p
_lib.mla_uses_tensor_cores.argtypes = [C.POINTER(Dims), C.c_int32]
_lib.mla_uses_tensor_cores.restype = C.c_int32
_lib.mla_kernel_launches.restype = C.c_uint64
for _f in ("mla_cache_append", "mla_absorb_q", "mla_decode", "mla_decode_noalloc", "mla_out_proj", "mla_o_proj",
           "mla_get_device_error", "mla_set_launch_overlap", "mla_get_launch_overlap", "mla_absorb_wo",
           "mla_o_proj_latent", "mla_absorb_merge", "mla_absorb_q_merged", "mla_front_end", "mla_selftest_timeout",
           "mla_query_heads", "mla_attend_order_a"):
    getattr(_lib, _f).restype = C.c_int


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.mla_last_error_message().decode()
        super().__init__(f"{where}: {_lib.mla_status_string(status).decode()}: {msg}")


def _check(status: int, where: str) -> None:
    if status != MLA_OK:
        raise MlaError(status, where)


def dims(d, n_h, d_h, d_c, d_cq, d_r, rope_base=10000.0, softmax_scale=0.0, dtype="bf16") -> Dims:
    return Dims(int(d), int(n_h), int(d_h), int(d_c), int(d_cq), int(d_r), float(rope_base),
                float(softmax_scale), MLA_BF16 if dtype == "bf16" else MLA_FP32)


def _ptr(t):
    if t is None:
        return None
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


class Cache:
    """A latent cache held in a torch device tensor.

    contiguous: data [num_seqs][max_len][D]; paged: data [num_blocks][block_size][D]
    with block_table [num_seqs][max_blocks_per_seq] int32 on the device.
    """

    def __init__(self, data: torch.Tensor, block_table: torch.Tensor | None = None):
        assert data.is_cuda and data.is_contiguous()
        self.data = data
        self.block_table = block_table
        if block_table is None:
            self.desc = CacheDesc(data.data_ptr(), 0, 0, None, 0, data.shape[0], data.shape[1], 0)
        else:
            assert block_table.dtype == torch.int32 and block_table.is_cuda and block_table.is_contiguous()
            self.desc = CacheDesc(data.data_ptr(), 1, data.shape[1], block_table.data_ptr(),
                                  block_table.shape[1], block_table.shape[0], 0, data.shape[0])


def workspace_size(p: Dims, op: int, rows: int, n_q: int = 1, max_seq_len: int = 0, num_splits: int = 0) -> int:
    return int(_lib.mla_workspace_size(C.byref(p), op, rows, n_q, max_seq_len, num_splits))


def cache_capacity(cache: "Cache") -> int:
    """Longest sequence the cache can hold (the bound mla_decode sizes forced splits by)."""
    d = cache.desc
    return d.max_blocks_per_seq * d.block_size if d.paged else d.max_len


def _ws(p, op, rows, n_q, ws, max_seq_len=0, num_splits=0):
    need = workspace_size(p, op, rows, n_q, max_seq_len, num_splits)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    return ws, need if ws is None else ws.numel()


def uses_tensor_cores(p: Dims, op: int) -> bool:
    return bool(_lib.mla_uses_tensor_cores(C.byref(p), op))


def mla_cache_append(p: Dims, h, W_DKV, W_KR, seq_idx, positions, cache: Cache, ws=None, stream=None):
    T = h.shape[0]
    ws, nbytes = _ws(p, OP_APPEND, T, 1, ws)
    _check(_lib.mla_cache_append(C.byref(p), _ptr(h), _ptr(W_DKV), _ptr(W_KR), _ptr(seq_idx),
                                 _ptr(positions), T, C.byref(cache.desc), _ptr(ws), nbytes,
                                 _stream(stream)), "mla_cache_append")


def mla_absorb_q(p: Dims, h, W_DQ, W_UQ, W_QR, W_UK, positions, q, ws=None, stream=None):
    T = h.shape[0]
    ws, nbytes = _ws(p, OP_ABSORB, T, 1, ws)
    _check(_lib.mla_absorb_q(C.byref(p), _ptr(h), _ptr(W_DQ), _ptr(W_UQ), _ptr(W_QR), _ptr(W_UK),
                             _ptr(positions), T, _ptr(q), _ptr(ws), nbytes, _stream(stream)),
           "mla_absorb_q")


def mla_decode(p: Dims, q, cache: Cache, seq_lens, n_q, o_lat, lse=None, num_splits=0, ws=None,
               stream=None):
    B = seq_lens.shape[0]
    ws, nbytes = _ws(p, OP_DECODE, B, n_q, ws, cache_capacity(cache), num_splits)
    _check(_lib.mla_decode(C.byref(p), _ptr(q), C.byref(cache.desc), _ptr(seq_lens), B, n_q,
                           _ptr(o_lat), _ptr(lse), num_splits, _ptr(ws), nbytes, _stream(stream)),
           "mla_decode")


def mla_decode_noalloc(p: Dims, q, cache: Cache, seq_lens, n_q, o_lat, lse=None, stream=None):
    """mla_decode with the library's static scratch (at most 64 token rows; calls
    that may overlap in time race on the scratch)."""
    B = seq_lens.shape[0]
    _check(_lib.mla_decode_noalloc(C.byref(p), _ptr(q), C.byref(cache.desc), _ptr(seq_lens), B, n_q,
                                   _ptr(o_lat), _ptr(lse), _stream(stream)), "mla_decode_noalloc")


def mla_out_proj(p: Dims, o_lat, W_UV, o, ws=None, stream=None):
    T = o_lat.shape[0]
    ws, nbytes = _ws(p, OP_OUT_PROJ, T, 1, ws)
    _check(_lib.mla_out_proj(C.byref(p), _ptr(o_lat), _ptr(W_UV), T, _ptr(o), _ptr(ws), nbytes,
                             _stream(stream)), "mla_out_proj")


def mla_o_proj(p: Dims, o, W_O, y, ws=None, stream=None):
    T = o.shape[0]
    ws, nbytes = _ws(p, OP_O_PROJ, T, 1, ws)
    _check(_lib.mla_o_proj(C.byref(p), _ptr(o), _ptr(W_O), T, _ptr(y), _ptr(ws), nbytes, _stream(stream)),
           "mla_o_proj")


def mla_absorb_wo(p: Dims, W_O, W_UV, W_OV, stream=None):
    """W_OV[r][h d_c + j] = sum_i W_O[r][h d_h + i] W_UV[h d_h + i][j] (offline)."""
    _check(_lib.mla_absorb_wo(C.byref(p), _ptr(W_O), _ptr(W_UV), _ptr(W_OV), _stream(stream)), "mla_absorb_wo")


def mla_o_proj_latent(p: Dims, o_lat, W_OV, y, ws=None, stream=None):
    T = o_lat.shape[0]
    ws, nbytes = _ws(p, OP_O_PROJ_LATENT, T, 1, ws)
    _check(_lib.mla_o_proj_latent(C.byref(p), _ptr(o_lat), _ptr(W_OV), T, _ptr(y), _ptr(ws), nbytes,
                                  _stream(stream)), "mla_o_proj_latent")


def mla_absorb_merge(p: Dims, W_UQ, W_UK, W_UQK, stream=None):
    """W_UQK[h d_c + j][c] = sum_i W_UK[h d_h + i][j] W_UQ[h d_h + i][c] (offline)."""
    _check(_lib.mla_absorb_merge(C.byref(p), _ptr(W_UQ), _ptr(W_UK), _ptr(W_UQK), _stream(stream)),
           "mla_absorb_merge")


def mla_absorb_q_merged(p: Dims, h, W_DQ, W_UQK, W_QR, positions, q, ws=None, stream=None):
    T = h.shape[0]
    ws, nbytes = _ws(p, OP_ABSORB_MERGED, T, 1, ws)
    _check(_lib.mla_absorb_q_merged(C.byref(p), _ptr(h), _ptr(W_DQ), _ptr(W_UQK), _ptr(W_QR), _ptr(positions), T,
                                    _ptr(q), _ptr(ws), nbytes, _stream(stream)), "mla_absorb_q_merged")


def mla_front_end(p: Dims, h, W_DKV, W_KR, W_DQ, W_UQ, W_QR, W_UK, seq_idx, positions, cache: Cache, q, ws=None,
                  stream=None):
    T = h.shape[0]
    ws, nbytes = _ws(p, OP_FRONT_END, T, 1, ws)
    _check(_lib.mla_front_end(C.byref(p), _ptr(h), _ptr(W_DKV), _ptr(W_KR), _ptr(W_DQ), _ptr(W_UQ), _ptr(W_QR),
                              _ptr(W_UK), _ptr(seq_idx), _ptr(positions), T, C.byref(cache.desc), _ptr(q), _ptr(ws),
                              nbytes, _stream(stream)), "mla_front_end")


def cache_rows(cache: "Cache") -> int:
    """Physical rows of the cache (the size mla_attend_order_a decompresses)."""
    d = cache.desc
    return d.num_blocks * d.block_size if d.paged else d.num_seqs * d.max_len


def mla_query_heads(p: Dims, h, W_DQ, W_UQ, W_QR, positions, qa, ws=None, stream=None):
    T = h.shape[0]
    ws, nbytes = _ws(p, OP_QUERY_HEADS, T, 1, ws)
    _check(_lib.mla_query_heads(C.byref(p), _ptr(h), _ptr(W_DQ), _ptr(W_UQ), _ptr(W_QR), _ptr(positions), T, _ptr(qa),
                                _ptr(ws), nbytes, _stream(stream)), "mla_query_heads")


def mla_attend_order_a(p: Dims, qa, W_UK, W_UV, cache: Cache, seq_lens, n_q, o, ws=None, stream=None):
    B = seq_lens.shape[0]
    ws, nbytes = _ws(p, OP_ATTEND_A, B, n_q, ws, cache_rows(cache))
    _check(_lib.mla_attend_order_a(C.byref(p), _ptr(qa), _ptr(W_UK), _ptr(W_UV), C.byref(cache.desc), _ptr(seq_lens),
                                   B, n_q, _ptr(o), _ptr(ws), nbytes, _stream(stream)), "mla_attend_order_a")


def mla_selftest_timeout(wait_ns: int, scratch, stream=None):
    """Launch the failure-path self-test (a kernel whose bounded wait runs out)."""
    _check(_lib.mla_selftest_timeout(int(wait_ns), _ptr(scratch), scratch.numel() * scratch.element_size(),
                                     _stream(stream)), "mla_selftest_timeout")


def mla_get_device_error(stream=None) -> int:
    """Synchronise the stream; return (and clear) the device error status."""
    return int(_lib.mla_get_device_error(_stream(stream)))


def status_string(s: int) -> str:
    return _lib.mla_status_string(s).decode()


def set_launch_overlap(enable: bool) -> None:
    """Process-wide: launch the tensor-core kernels with programmatic stream
    serialization, so that each may set up and start streaming its weights
    while the kernel ahead of it finishes (results are identical). The weights
    of a call must not be written by the work enqueued just before it."""
    _check(_lib.mla_set_launch_overlap(1 if enable else 0), "mla_set_launch_overlap")


def get_launch_overlap() -> bool:
    return bool(_lib.mla_get_launch_overlap())


def kernel_launches() -> int:
    """Kernels launched by the library so far in this process."""
    return int(_lib.mla_kernel_launches())
