"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle
on the same seeded inputs.  Needs a B200 (sm_100a)."""
import numpy as np
import pytest
import torch

import exact_io_aware_78_b200 as ea
from exact_io_aware_78_b200 import _binding as Bn
from exact_io_aware_78_b200.inputs import WORKLOADS, make_inputs, make_ramp_inputs, sample_rows, workload_inputs
from oracle import attention_ref

from gpu_helpers import assert_close, case, oracle_view, ranges_view, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(lib_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    major, _ = torch.cuda.get_device_capability(0)
    if major != 10:
        pytest.skip("needs an sm_100 GPU")
    torch.cuda.set_device(0)
    ea.load_library(lib_path)
    yield


# --------------------------------------------------------------- small shapes
# Element-by-element over all outputs: several tiles, ragged tails, the
# degenerate N = 1, masks, GQA groups 1..8, both head dims.
SMALL = [
    # B, Hq, Hkv, N, d, causal, window, dtype
    (1, 1, 1, 128, 128, False, 0, "bf16"),
    (1, 1, 1, 128, 64, False, 0, "bf16"),
    (1, 1, 1, 1, 128, True, 0, "bf16"),
    (1, 2, 1, 1, 64, False, 0, "bf16"),
    (1, 1, 1, 17, 64, False, 0, "bf16"),
    (3, 2, 1, 127, 128, True, 0, "bf16"),
    (1, 2, 2, 129, 128, False, 0, "bf16"),
    (2, 3, 3, 200, 128, True, 0, "bf16"),
    (1, 4, 2, 257, 64, True, 0, "bf16"),
    (1, 8, 1, 384, 128, True, 0, "bf16"),
    (1, 2, 2, 300, 128, True, 100, "bf16"),
    (1, 1, 1, 600, 128, True, 128, "bf16"),
    (1, 1, 1, 600, 128, True, 1, "bf16"),
    (1, 2, 1, 520, 64, False, 200, "bf16"),
    (1, 8, 2, 1000, 128, True, 0, "bf16"),
    (1, 2, 2, 1024, 128, True, 0, "bf16"),
    (1, 2, 2, 300, 128, True, 0, "fp8"),
    (1, 2, 1, 513, 128, False, 0, "fp8"),
    (1, 2, 2, 700, 128, True, 256, "fp8"),
    (1, 1, 1, 128, 64, False, 0, "fp32"),
    (2, 2, 1, 300, 64, True, 50, "fp32"),
    (1, 3, 3, 1, 64, True, 0, "fp32"),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,window,dtype", SMALL,
                         ids=[f"B{c[0]}h{c[1]}kv{c[2]}n{c[3]}d{c[4]}c{int(c[5])}w{c[6]}{c[7]}" for c in SMALL])
def test_small_shapes(B, Hq, Hkv, N, d, causal, window, dtype):
    case(B, Hq, Hkv, N, d, causal, window, dtype, seed=1000 + N + d + Hq)


def test_sharpened_queries_stress_rescale():
    """Q x 4: logits spread widely, the running max moves often and the lazy
    rescale of O fires."""
    case(1, 4, 4, 777, 128, True, 0, "bf16", seed=77, q_mult=4.0)
    case(1, 2, 2, 512, 128, False, 0, "bf16", seed=78, q_mult=4.0)


def _reference_moves(q, k, causal, scale, tau):
    """How often each row's reference maximum must move under the kernel's
    rule (set by the row's first visible 128-key tile, moved when a later
    tile's maximum exceeds it by more than tau, in log2 units)."""
    cs = scale / np.log(2.0)
    s = np.einsum("bihd,bjhd->bhij", q, k) * cs
    N = s.shape[-1]
    if causal:
        s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
    tm = np.stack([s[..., j:j + 128].max(-1) for j in range(0, N, 128)], -1)
    ref = tm[..., 0].copy()
    moves = np.zeros(ref.shape, int)
    for t in range(1, tm.shape[-1]):
        up = tm[..., t] > ref + tau
        moves += up
        ref = np.where(up, tm[..., t], ref)
    return moves


@pytest.mark.parametrize("dtype,tau", [("bf16", 16.0), ("fp8", 8.0)])
@pytest.mark.parametrize("causal", [True, False])
def test_growing_scores_move_the_reference(dtype, tau, causal):
    """Scores that grow along the keys make every row's reference maximum
    move several times, so the rescale of l and O (and, for the first half of
    a tile computed against the old reference, its recomputation) runs on
    most steps; the result must still match the oracle."""
    B, H, N, d = 1, 2, 1000, 128
    inp = make_ramp_inputs(B, H, N, d, dtype, 4040 + causal, ramp=8.0)
    q, k, v = oracle_view(inp, dtype)
    moves = _reference_moves(q, k, causal, d ** -0.5, tau)
    rows_seen = moves[..., 256:]  # rows that see at least three tiles
    assert np.median(rows_seen) >= 2, "inputs do not exercise the rescale path"
    O, L = run_gpu(inp, causal, 0, d ** -0.5)
    Oref, Lref = attention_ref(q, k, v, causal, 0, d ** -0.5)
    assert_close(O, L, Oref, Lref, dtype, f"growing scores {dtype} causal={causal}")


# --------------------------------------------------------- full workloads
@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_sampled_rows(name):
    """Each workload at its full size, launched exactly as the benchmark
    launches it; the oracle evaluates a seeded sample of rows (plus the
    first/last rows, tile edges and window edges) for every (b, h)."""
    w = WORKLOADS[name]
    rows = sample_rows(w.N, w.window, 48, seed=w.seed) if w.N > 512 else None
    inp = workload_inputs(w)
    O, L = run_gpu(inp, w.causal, w.window, w.scale)
    # properties that hold at any size
    assert np.isfinite(O).all() and np.isfinite(L).all()
    q, k, v = oracle_view(inp, w.dtype)
    lo, hi = ranges_view(inp)
    Oref, Lref = attention_ref(q, k, v, w.causal, w.window, w.scale, rows=rows, key_lo=lo, key_hi=hi)
    if rows is not None:
        O, L = O[:, rows], L[:, :, rows]
    assert_close(O, L, Oref, Lref, w.dtype, name)


# ------------------------------------------------------ kernel invariants
def _run_raw(inp, causal, window):
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    o, lse = ea.forward(q, k, v, causal=causal, window=window)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def test_deterministic_and_schedule_independent():
    """Bitwise-equal results across repeated runs, tile orders and CTA
    counts (each query tile's reduction order is fixed by the key order)."""
    inp = make_inputs(2, 4, 2, 1100, 128, "bf16", 5)
    ref = _run_raw(inp, True, 0)
    try:
        for order, ctas in [(0, 0), (1, 0), (0, 1), (1, 3), (0, 7)]:
            ea.attn_set_option(Bn.EA_OPT_SCHEDULE_ORDER, order)
            ea.attn_set_option(Bn.EA_OPT_MAX_CTAS, ctas)
            o, l = _run_raw(inp, True, 0)
            assert torch.equal(o, ref[0]) and torch.equal(l, ref[1]), (order, ctas)
    finally:
        ea.attn_set_option(Bn.EA_OPT_SCHEDULE_ORDER, 0)
        ea.attn_set_option(Bn.EA_OPT_MAX_CTAS, 0)


def test_batch_position_independent():
    """A (b, h) slice gives the same bits whether it runs alone or inside a
    larger batch."""
    inp = make_inputs(3, 2, 2, 333, 128, "bf16", 9)
    o_all, l_all = _run_raw(inp, True, 0)
    one = {n: inp[n][1:2].contiguous() if inp[n] is not None else None for n in inp}
    o1, l1 = _run_raw(one, True, 0)
    assert torch.equal(o_all[1:2], o1) and torch.equal(l_all[1:2], l1)


def test_outputs_stay_inside_their_buffers():
    """Guard regions around O and LSE keep their fill pattern."""
    dev = torch.device("cuda:0")
    B, Hq, Hkv, N, d = 1, 3, 1, 333, 128
    inp = make_inputs(B, Hq, Hkv, N, d, "bf16", 11)
    q, k, v = (inp[n].to(dev) for n in "qkv")
    G = 4096
    n_o = B * N * Hq * d
    n_l = B * Hq * N
    o_buf = torch.full((G + n_o + G,), -7.0, device=dev, dtype=torch.bfloat16)
    l_buf = torch.full((G + n_l + G,), -7.0, device=dev, dtype=torch.float32)
    o = o_buf[G:G + n_o].view(B, N, Hq, d)
    lse = l_buf[G:G + n_l].view(B, Hq, N)
    ea.attn_fwd(q, k, v, o, lse, causal=True)
    torch.cuda.synchronize()
    assert torch.all(o_buf[:G] == -7.0) and torch.all(o_buf[G + n_o:] == -7.0)
    assert torch.all(l_buf[:G] == -7.0) and torch.all(l_buf[G + n_l:] == -7.0)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_bounded_wait_reports_timeout_and_context_survives():
    """The load warp skips one copy, so a consumer's bounded wait runs out:
    the launch reports EA_EDEVICE_TIMEOUT with the failing site, nothing
    traps, and the next launch on the same context is correct."""
    inp = make_inputs(1, 2, 2, 512, 128, "bf16", 13)
    try:
        ea.attn_set_option(Bn.EA_OPT_WAIT_TIMEOUT_NS, 50_000_000)
        ea.attn_set_option(Bn.EA_OPT_SKIP_ARRIVE_ONCE, 1)
        dev = torch.device("cuda:0")
        q, k, v = (inp[n].to(dev) for n in "qkv")
        ea.forward(q, k, v, causal=True)
        st, code, site = ea.attn_get_last_error()
        assert st == Bn.EA_EDEVICE_TIMEOUT and code == 1 and site > 0, (st, code, site)
        st2, _, _ = ea.attn_get_last_error()
        assert st2 == 0  # the word was cleared
    finally:
        ea.attn_set_option(Bn.EA_OPT_WAIT_TIMEOUT_NS, 2_000_000_000)
        ea.attn_set_option(Bn.EA_OPT_SKIP_ARRIVE_ONCE, 0)
    case(1, 2, 2, 512, 128, True, 0, "bf16", seed=13)


def test_host_pointer_rejected():
    """A host (pageable) buffer is refused before anything is queued."""
    lib = ea.load_library()
    dev = torch.device("cuda:0")
    q = torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16, device=dev)
    host = torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 128, device=dev)
    rc = lib.attn_fwd(q.data_ptr(), host.data_ptr(), q.data_ptr(), q.data_ptr(), lse.data_ptr(), 1, 1, 1, 128,
                      128, 0, 0, 0.1, Bn.EA_BF16, None, None, None, None)
    assert rc == Bn.EA_EINVAL
