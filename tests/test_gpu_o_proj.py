"""Output projection y = W_O o (MLA walk-through, section 1 step 5) through
the C ABI against the fp64 oracle, element by element: DeepSeek-V2 dims on
the tensor cores (split-K GEMM + finalize; several tiles and a ragged token
tail, up to 200 token rows) and the tiny dims on the CUDA cores in fp32 and
bf16 storage."""
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


TINY_BF16 = synth.shrink(synth.WORKLOADS["tiny_fp32"], dtype="bf16")


@pytest.mark.parametrize("name,T", [("v2_b64_paged", 1), ("v2_b64_paged", 37), ("v2_b64_paged", 64),
                                    ("v2_b64_paged", 200), ("tiny_fp32", 5), ("tiny_bf16", 7)])
def test_o_proj_matches_oracle(mla, name, T):
    import torch
    import oracle as orc
    from tests.gpu_util import assert_close, dev, dims_of, host
    w = TINY_BF16 if name == "tiny_bf16" else synth.WORKLOADS[name]
    p = dims_of(w, mla)
    assert mla.uses_tensor_cores(p, mla.OP_O_PROJ) == (name == "v2_b64_paged")
    HD = w.n_h * w.d_h
    rng = np.random.default_rng(4242 + T)
    W_O = rng.standard_normal((w.d, HD), dtype=np.float32) / np.float32(np.sqrt(HD))
    o = rng.standard_normal((T, HD), dtype=np.float32)
    if w.dtype == "bf16":
        W_bits, o_bits = synth.bf16_bits(W_O), synth.bf16_bits(o)
        W_O, o = synth.bf16_to_f32(W_bits), synth.bf16_to_f32(o_bits)
        W_d, o_d = dev(W_bits, "bf16"), dev(o_bits, "bf16")
        y = torch.empty((T, w.d), device="cuda", dtype=torch.bfloat16)
    else:
        W_d, o_d = torch.from_numpy(W_O).cuda(), torch.from_numpy(o).cuda()
        y = torch.empty((T, w.d), device="cuda", dtype=torch.float32)
    mla.mla_o_proj(p, o_d, W_d, y)
    assert mla.mla_get_device_error() == mla.MLA_OK
    ref = orc.o_proj(W_O.astype(np.float64), o.astype(np.float64))
    assert_close(host(y), ref, "y = W_O o")
