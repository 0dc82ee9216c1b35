"""Pins for the backward oracle (dQ, dK, dV of the exact attention).  Each
pin ties it to something other than itself: central finite differences of the
forward oracle, torch's float64 autograd, the algebra of the softmax Jacobian
(rows of dS sum to zero), closed forms for keys nobody sees, and the GQA
reduction to repeated heads.  The mutation tests plant plausible slips in a
copy of the oracle's source and check that a pin catches each.  CPU only."""
import inspect
import textwrap

import numpy as np
import pytest
import torch

import oracle.backward as ob
from oracle import attention_ref, probabilities_ref
from exact_io_aware_78_b200.inputs import make_row_ranges

RNG = np.random.default_rng(77)


def rand(*shape):
    return RNG.standard_normal(shape)


BWD = {"f": ob.attention_bwd_ref}


def bwd(*a, **kw):
    return BWD["f"](*a, **kw)


def loss(q, k, v, g, causal, window, lo, hi):
    o, _ = attention_ref(q, k, v, causal, window, key_lo=lo, key_hi=hi)
    return float((o * g).sum())


# ---------------------------------------------------------------- pins

def pin_finite_differences():
    """dL/dX by central differences of the forward oracle, L = sum(O * dO),
    for causal, windowed, row-range (with empty rows) and GQA cases."""
    B, N, Hq, Hkv, d = 1, 6, 2, 1, 3
    cases = [(False, 0, None, None), (True, 0, None, None), (True, 3, None, None),
             (False, 0, np.array([[2, 0, 5, 1, 3, 0]]), np.array([[5, 2, 5, 6, 4, 6]])),
             (True, 0, np.array([[0, 0, 1, 3, 2, 0]]), np.array([[1, 0, 3, 6, 4, 6]]))]
    for causal, window, lo, hi in cases:
        q, k, v, g = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d), rand(B, N, Hq, d)
        dq, dk, dv = bwd(q, k, v, g, causal, window, key_lo=lo, key_hi=hi)
        eps = 1e-6
        for x, dx in ((q, dq), (k, dk), (v, dv)):
            it = np.nditer(x, flags=["multi_index"])
            for _ in it:
                ix = it.multi_index
                old = x[ix]
                x[ix] = old + eps
                lp = loss(q, k, v, g, causal, window, lo, hi)
                x[ix] = old - eps
                lm = loss(q, k, v, g, causal, window, lo, hi)
                x[ix] = old
                assert abs((lp - lm) / (2 * eps) - dx[ix]) < 1e-7, (causal, window, ix)


def pin_torch_autograd():
    """torch float64 autograd through softmax(scale Q K^T + mask) V with an
    explicit boolean mask (rows with at least one visible key), GQA by
    repeating the key/value heads."""
    B, N, Hq, Hkv, d = 2, 20, 4, 2, 8
    for causal, window, kind in [(True, 0, None), (False, 0, "documents"), (True, 5, None)]:
        q, k, v, g = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d), rand(B, N, Hq, d)
        lo = hi = None
        if kind:
            lo, hi = (t.numpy() for t in make_row_ranges(kind, B, N, 3, 3, 9))
        dq, dk, dv = bwd(q, k, v, g, causal, window, key_lo=lo, key_hi=hi)
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        i = torch.arange(N).view(N, 1)
        j = torch.arange(N).view(1, N)
        m = torch.ones(B, N, N, dtype=torch.bool)
        if causal:
            m &= j <= i
        if window > 0:
            m &= j > i - window
        if lo is not None:
            m &= (j >= torch.from_numpy(lo).view(B, N, 1)) & (j < torch.from_numpy(hi).view(B, N, 1))
        assert m.any(-1).all()
        kr = tk.repeat_interleave(Hq // Hkv, dim=2)
        vr = tv.repeat_interleave(Hq // Hkv, dim=2)
        s = torch.einsum("bihc,bjhc->bhij", tq, kr) / np.sqrt(d)
        s = s.masked_fill(~m.unsqueeze(1), float("-inf"))
        o = torch.einsum("bhij,bjhc->bihc", torch.softmax(s, -1), vr)
        (o * torch.tensor(g)).sum().backward()
        np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
        np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
        np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12)


def pin_softmax_jacobian_rows_sum_to_zero():
    """Rows of dS sum to zero, so dK sums to zero over all keys of each
    (b, kv head); P rows sum to one, so dV sums to the sum of dO over the
    group's rows that see a key.  Also D = rowsum(dO o O) = rowsum(P o dP)."""
    B, N, Hq, Hkv, d = 2, 15, 4, 2, 6
    lo, hi = (t.numpy() for t in make_row_ranges("random", B, N, 5))
    q, k, v, g = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d), rand(B, N, Hq, d)
    dq, dk, dv = bwd(q, k, v, g, True, 0, key_lo=lo, key_hi=hi)
    o, lse = attention_ref(q, k, v, True, 0, key_lo=lo, key_hi=hi)
    has = np.isfinite(lse)  # [B, Hq, N]
    for b in range(B):
        for kh in range(Hkv):
            np.testing.assert_allclose(dk[b, :, kh].sum(axis=0), 0.0, atol=1e-12)
            heads = range(kh * 2, kh * 2 + 2)
            want = sum(g[b, has[b, h], h].sum(axis=0) for h in heads)
            np.testing.assert_allclose(dv[b, :, kh].sum(axis=0), want, atol=1e-12)
    P = probabilities_ref(q, k, True, 0, key_lo=lo, key_hi=hi)
    for b in range(B):
        for h in range(Hq):
            dp = g[b, :, h] @ v[b, :, h // 2].T
            np.testing.assert_allclose((P[b, h] * dp).sum(axis=1), (g[b, :, h] * o[b, :, h]).sum(axis=1),
                                       atol=1e-12)


def pin_unseen_keys_get_zero_gradient():
    """Keys that no query may see get dK = dV = 0; queries that see no key
    get dQ = 0."""
    B, N, H, d = 1, 10, 2, 4
    q, k, v, g = rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d)
    lo = np.full((B, N), 3)
    hi = np.full((B, N), 7)
    hi[0, 8] = 3                       # row 8 sees nothing
    dq, dk, dv = bwd(q, k, v, g, False, 0, key_lo=lo, key_hi=hi)
    assert np.all(dk[:, :3] == 0) and np.all(dk[:, 7:] == 0)
    assert np.all(dv[:, :3] == 0) and np.all(dv[:, 7:] == 0)
    assert np.all(dq[:, 8] == 0)
    assert np.abs(dk[:, 3:7]).max() > 0 and np.abs(dv[:, 3:7]).max() > 0


def pin_gqa_is_repeated_heads_summed():
    B, N, Hq, Hkv, d = 1, 9, 6, 2, 5
    q, k, v, g = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d), rand(B, N, Hq, d)
    dq, dk, dv = bwd(q, k, v, g, True, 0)
    kr, vr = np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2)
    dq2, dk2, dv2 = bwd(q, kr, vr, g, True, 0)
    np.testing.assert_allclose(dq, dq2, atol=1e-13)
    np.testing.assert_allclose(dk, dk2.reshape(B, N, Hkv, 3, d).sum(axis=3), atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, N, Hkv, 3, d).sum(axis=3), atol=1e-13)


def pin_given_forward_outputs_are_used():
    """Passing the forward's O and LSE gives the same gradients as letting
    the oracle recompute them."""
    q, k, v, g = rand(1, 11, 2, 4), rand(1, 11, 2, 4), rand(1, 11, 2, 4), rand(1, 11, 2, 4)
    o, lse = attention_ref(q, k, v, True, 4)
    a = bwd(q, k, v, g, True, 4)
    b = bwd(q, k, v, g, True, 4, o=o, lse=lse)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-14)


PINS = [pin_finite_differences, pin_torch_autograd, pin_softmax_jacobian_rows_sum_to_zero,
        pin_unseen_keys_get_zero_gradient, pin_gqa_is_repeated_heads_summed, pin_given_forward_outputs_are_used]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_shape_checks():
    q = rand(1, 4, 2, 3)
    with pytest.raises(ValueError):
        ob.attention_bwd_ref(q, q[:, :, :1], q[:, :, :1], q[:, :3])


# ---------------------------------------------------------------- mutants
# Each mutant is the oracle's own source with one line changed, compiled in
# the oracle module's namespace.
MUTANTS = {
    "no_D_term": ("ds = p * (dp - D)", "ds = p * dp"),
    "dV_not_transposed": ("dv[b, :, kh] += p.T @ dob", "dv[b, :, kh] += p @ dob"),
    "dQ_scale_dropped": ("dq[b, :, h] = scale * (ds @ kb)", "dq[b, :, h] = ds @ kb"),
    "D_from_dO_only": ("D = (dob * o[b, :, h]).sum(axis=1, keepdims=True)", "D = dob.sum(axis=1, keepdims=True)"),
    "gqa_dK_overwritten": ("dk[b, :, kh] += scale * (ds.T @ qb)", "dk[b, :, kh] = scale * (ds.T @ qb)"),
    "mask_ignored": ("p = np.where(ok & fin[:, None], np.exp(s - ref), 0.0)",
                     "p = np.where(fin[:, None], np.exp(s - ref), 0.0)"),
}


def _mutant(old, new):
    src = textwrap.dedent(inspect.getsource(ob.attention_bwd_ref))
    assert src.count(old) == 1, old
    ns = dict(vars(ob))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns["attention_bwd_ref"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    monkeypatch.setitem(BWD, "f", _mutant(*MUTANTS[name]))
    caught = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
