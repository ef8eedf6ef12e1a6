"""The oracle's pins catch plausible mistakes: each case below plants one
mistake in a copy of the oracle's C source (a flipped sign, a dropped term, a
transposed or misplaced index, a wrong constant), builds the copy, and
requires at least one pin of tests/test_oracle_pins.py to fail against it. The
oracle itself is never modified; every planted mistake keeps all memory
accesses in bounds."""
import ctypes as C
import inspect
import os
import subprocess

import pytest

import oracle as orc
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(orc.__file__), "mla_oracle.c")

# (name, text in the oracle, replacement)
MUTANTS = [
    ("rope rotation sign", "x[2 * i] = x0 * c - x1 * s;", "x[2 * i] = x0 * c + x1 * s;"),
    ("rope frequency exponent", "pow(base, -2.0 * (double)i / (double)d_r)", "pow(base, -1.0 * (double)i / (double)d_r)"),
    ("rope pair order", "double x0 = x[2 * i], x1 = x[2 * i + 1];", "double x1 = x[2 * i], x0 = x[2 * i + 1];"),
    ("softmax scale without d_R", "1.0 / sqrt((double)(p->d_h + p->d_r))", "1.0 / sqrt((double)(p->d_h))"),
    ("score drops the RoPE term",
     "for (int j = 0; j < D; ++j) acc += q[j] * orc_read(c->data, c->dtype, row * D + j);",
     "for (int j = 0; j < p->d_c; ++j) acc += q[j] * orc_read(c->data, c->dtype, row * D + j);"),
    ("W_UK read transposed", "acc += W_UK[((int64_t)hh * p->d_h + i) * p->d_c + j] * qc[i];",
     "acc += W_UK[(int64_t)hh * p->d_h * p->d_c + (int64_t)j * p->d_h + i] * qc[i];"),
    ("query RoPE at the wrong position", "orc_rope(q + p->d_c, p->d_r, (double)positions[t], p->rope_base);",
     "orc_rope(q + p->d_c, p->d_r, (double)positions[t] + 1.0, p->rope_base);"),
    ("key RoPE skipped", "orc_rope(out + p->d_c, p->d_r, (double)positions[t], p->rope_base);", ";"),
    ("causal range one short", "return (int64_t)seq_lens[b] - n_q + 1 + j;", "return (int64_t)seq_lens[b] - n_q + j;"),
    ("softmax not normalised", "double w = exp(scores[i - start] - m) / z;", "double w = exp(scores[i - start] - m);"),
    ("lse without the max", "*lse = m + log(z);", "*lse = log(z);"),
    ("combine weight inverted", "double w = exp(lse_parts[s] - L);", "double w = exp(L - lse_parts[s]);"),
    ("out-projection uses head 0 for every head", "orc_matvec(W_UV + (int64_t)hh * p->d_h * p->d_c, p->d_h, p->d_c,",
     "orc_matvec(W_UV, p->d_h, p->d_c,"),
    ("bf16 bits shifted", "uint32_t u = ((uint32_t)b) << 16;", "uint32_t u = ((uint32_t)b) << 15;"),
    ("paged slot ignores the block offset", "return blk * c->block_size + pos % c->block_size;",
     "return blk * c->block_size;"),
    ("W_O absorption reads W_UV transposed",
     "acc += W_O[r * ko + (int64_t)hh * p->d_h + i] * W_UV[((int64_t)hh * p->d_h + i) * p->d_c + j];",
     "acc += W_O[r * ko + (int64_t)hh * p->d_h + i] * W_UV[(int64_t)hh * p->d_h * p->d_c + (int64_t)j * p->d_h + i];"),
    ("merged absorption reads W_UQ transposed",
     "acc += W_UK[((int64_t)hh * p->d_h + i) * p->d_c + j] * W_UQ[((int64_t)hh * p->d_h + i) * p->d_cq + c];",
     "acc += W_UK[((int64_t)hh * p->d_h + i) * p->d_c + j] * W_UQ[(int64_t)hh * p->d_h * p->d_cq + (int64_t)c * p->d_h + i];"),
    ("merged absorption drops the last head row",
     "        for (int i = 0; i < p->d_h; ++i)\n          acc += W_UK[((int64_t)hh * p->d_h + i) * p->d_c + j] * W_UQ",
     "        for (int i = 0; i < p->d_h - 1; ++i)\n          acc += W_UK[((int64_t)hh * p->d_h + i) * p->d_c + j] * W_UQ"),
    ("order A decompresses values with W_UK",
     "        orc_matvec(Wv, p->d_h, p->d_c, ckv, v);", "        orc_matvec(Wk, p->d_h, p->d_c, ckv, v);"),
    ("order A reads every head's values from head 0",
     "const double *Wv = W_UV + hh * (int64_t)p->d_h * p->d_c;", "const double *Wv = W_UV;"),
    ("order A drops the RoPE term",
     "          acc += qr[jj] * orc_read(c->data, c->dtype, row * D + p->d_c + jj);",
     "          acc += 0.0 * qr[jj];"),
    ("order A softmax not normalised", "double w = exp(scores[i] - m) / z;", "double w = exp(scores[i] - m);"),
    ("output projection skips a token row",
     "for (int t = 0; t < T; ++t) orc_matvec(W, rows, cols, x + (int64_t)t * cols, y + (int64_t)t * rows);",
     "for (int t = 0; t < T; ++t) orc_matvec(W, rows, cols, x + (int64_t)(t > 0 ? t - 1 : 0) * cols, y + (int64_t)t * rows);"),
]


def _pin_functions():
    fns = [f for name, f in inspect.getmembers(pins, inspect.isfunction)
           if name.startswith("test_") and "orc" in inspect.signature(f).parameters]
    # cheapest first: the first failing pin ends a case
    return sorted(fns, key=lambda f: f.__name__ == "test_mla_reduces_to_mha")


@pytest.fixture(scope="module")
def pristine():
    orc.lib()
    return open(SRC).read()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_a_planted_mistake_fails_a_pin(pristine, tmp_path, name, old, new):
    assert pristine.count(old) == 1, f"mutation site not found once: {old}"
    src = tmp_path / "mutant.c"
    src.write_text(pristine.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(src), "-lm"])
    mutant = orc.bind(C.CDLL(str(so)))
    saved = orc._lib
    orc._lib = mutant
    caught = None
    try:
        for f in _pin_functions():
            try:
                f(orc)
            except Exception as e:  # noqa: BLE001 - a failing pin is the expected outcome
                caught = (f.__name__, type(e).__name__)
                break
    finally:
        orc._lib = saved
    assert caught is not None, f"no pin fails when the oracle has this mistake: {name}"
