"""Helpers shared by the GPU parity tests: device upload and the tolerance check."""
import numpy as np
import torch

from mla_latent_kv_33_b200 import synth

# |gpu - ref| <= ATOL + RTOL * |ref| per output element (bf16 storage, fp32 accumulation)
ATOL = 1e-2
RTOL = 1e-2


def dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Upload storage-format data: uint16 bf16 bits or float32 values."""
    if dtype == "bf16":
        assert x.dtype == np.uint16
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def store(inp_vals, inp_bits, dtype):
    return dev(inp_bits if dtype == "bf16" else inp_vals, dtype)


def host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def cache_host(t: torch.Tensor, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def assert_close(gpu, ref, what, atol=ATOL, rtol=RTOL):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    err = np.abs(gpu - ref)
    bound = atol + rtol * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - bound, -np.inf)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} elements out of tolerance; worst at {i}: "
                             f"gpu={gpu[i]!r} ref={ref[i]!r} err={err[i]:.3e} bound={bound[i]:.3e}")


def dims_of(w: synth.Workload, mla):
    return mla.dims(w.d, w.n_h, w.d_h, w.d_c, w.d_cq, w.d_r, w.rope_base, 0.0, w.dtype)


def orc_dims_of(w: synth.Workload, orc):
    return orc.dims(w.d, w.n_h, w.d_h, w.d_c, w.d_cq, w.d_r, w.rope_base)
