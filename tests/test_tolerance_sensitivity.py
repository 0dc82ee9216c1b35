"""The GPU parity bars are tight enough to catch a broken rescale: mistakes
are planted in a copy of the blockwise oracle (on the CPU, 128-key blocks as
the kernel's tiles) and its outputs, on inputs whose running maximum climbs
from tile to tile, must fail the bars the GPU tests apply; the unmodified
blockwise oracle must pass them.  The same inputs drive the GPU test that
moves the kernel's reference maximum."""
import inspect
import textwrap

import numpy as np
import pytest
import torch

from exact_io_aware_78_b200.inputs import make_ramp_inputs
from oracle import attention as oa
from oracle import attention_ref, dequantize_per_head

from gpu_helpers import TOL, errors

MUTANTS = {
    # the running output is not rescaled when the running maximum moves
    "output_rescale_dropped": ("acc = alpha[:, None] * acc + p @ vb_all[cols]", "acc = acc + p @ vb_all[cols]"),
    # the running sum is not rescaled
    "sum_rescale_dropped": ("l = alpha * l + p.sum(axis=1)", "l = l + p.sum(axis=1)"),
    # the rescale factor is applied the wrong way round
    "rescale_inverted": ("acc = alpha[:, None] * acc + p @ vb_all[cols]",
                         "acc = acc / np.where(alpha > 0, alpha, 1.0)[:, None] + p @ vb_all[cols]"),
}


def _mutant(old, new):
    src = textwrap.dedent(inspect.getsource(oa.online_ref))
    assert src.count(old) == 1, old
    ns = dict(vars(oa))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns["online_ref"]


def _inputs(dtype, causal):
    inp = make_ramp_inputs(1, 1, 512, 128, dtype, 4040 + causal, ramp=8.0)
    if dtype == "fp8":
        return tuple(dequantize_per_head(inp[n].view(torch.uint8).numpy(), inp[n + "_scale"].numpy()) for n in "qkv")
    return tuple(inp[n].to(torch.float64).numpy() for n in "qkv")


def _fails_bars(O, L, Oref, Lref, dtype):
    mx, mean, lse = errors(O, L, Oref, Lref)
    tmax, tmean, tlse = TOL[dtype]
    return not (np.isfinite(O).all() and mx <= tmax and mean <= tmean and lse <= tlse)


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("causal", [True, False])
def test_blockwise_oracle_passes_the_bars(dtype, causal):
    q, k, v = _inputs(dtype, causal)
    Oref, Lref = attention_ref(q, k, v, causal)
    O, L = oa.online_ref(q, k, v, causal, block_q=128, block_k=128)
    assert not _fails_bars(O, L, Oref, Lref, dtype)


@pytest.mark.parametrize("name", sorted(MUTANTS))
@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("causal", [True, False])
def test_bars_catch_a_broken_rescale(name, dtype, causal):
    q, k, v = _inputs(dtype, causal)
    Oref, Lref = attention_ref(q, k, v, causal)
    with np.errstate(all="ignore"):
        O, L = _mutant(*MUTANTS[name])(q, k, v, causal, block_q=128, block_k=128)
    assert _fails_bars(O, L, Oref, Lref, dtype), f"the bars do not catch {name}"
