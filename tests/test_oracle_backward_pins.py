"""Pins of the backward oracle against central finite differences of the forward
oracle (a property of derivatives, independent of the chain rule written out in
oracle/moe_backward.py), plus invariants; mutation tests at the end."""
import numpy as np
import pytest

from oracle import moe_backward as bwd
from oracle import moe_oracle as orc


def _problem(seed=0, shared=True, bias=True, selection=True):
    rng = np.random.default_rng(seed)
    T, d, N, k, f, fs = 12, 8, 5, 2, 6, 4
    p = dict(
        x=rng.normal(size=(T, d)),
        w_router=rng.normal(size=(d, N)) * 0.7,
        bias=rng.normal(size=N) * 0.3 if bias else None,
        w1=rng.normal(size=(N, d, f)) * 0.5,
        w3=rng.normal(size=(N, d, f)) * 0.5,
        w2=rng.normal(size=(N, f, d)) * 0.5,
        ws1=rng.normal(size=(d, fs)) * 0.5 if shared else None,
        ws3=rng.normal(size=(d, fs)) * 0.5 if shared else None,
        ws2=rng.normal(size=(fs, d)) * 0.5 if shared else None,
    )
    kw = dict(k=k, cap=4, align=8, aux_weight=0.3, z_weight=0.2,
              selection_bias=(rng.normal(size=N) * 0.2).astype(np.float32) if selection else None)
    dy = rng.normal(size=(T, d))
    return p, kw, dy


def _loss(p, kw, dy):
    return bwd.layer_loss(p["x"], p["w_router"], p["bias"], p["w1"], p["w3"], p["w2"], dy,
                          ws1=p["ws1"], ws3=p["ws3"], ws2=p["ws2"], **kw)


def _grads(p, kw, dy, b=bwd):
    return b.layer_backward(p["x"], p["w_router"], p["bias"], p["w1"], p["w3"], p["w2"], dy,
                            ws1=p["ws1"], ws3=p["ws3"], ws2=p["ws2"], **kw)


GRAD_OF = {"x": "dx", "w_router": "dw_router", "bias": "dbias", "w1": "dw1", "w3": "dw3", "w2": "dw2",
           "ws1": "dws1", "ws3": "dws3", "ws2": "dws2"}


def check_finite_differences(b=bwd, seed=0, n_coords=40, eps=1e-6):
    p, kw, dy = _problem(seed)
    g = _grads(p, kw, dy, b)
    L0, route0 = _loss(p, kw, dy)
    rng = np.random.default_rng(seed + 100)
    checked = 0
    for name, gname in GRAD_OF.items():
        P = p[name]
        G = getattr(g, gname)
        flat = P.reshape(-1)
        coords = rng.choice(flat.size, size=min(n_coords, flat.size), replace=False)
        for c in coords:
            old = flat[c]
            flat[c] = old + eps
            Lp, rp = _loss(p, kw, dy)
            flat[c] = old - eps
            Lm, rm = _loss(p, kw, dy)
            flat[c] = old
            if not all(np.array_equal(a, b_) for a, b_ in zip(rp + rm, route0 + route0)):
                continue                                   # routing changed: not differentiable here
            fd = (Lp - Lm) / (2 * eps)
            an = G.reshape(-1)[c]
            assert abs(fd - an) <= 1e-5 * max(1.0, abs(fd)), (name, c, fd, an)
            checked += 1
    assert checked >= 0.9 * sum(min(n_coords, p[n].size) for n in GRAD_OF), checked
    # the selection bias gets no gradient: the loss moves only where the routing changes
    sb = kw["selection_bias"]
    for i in range(len(sb)):
        old = sb[i]
        sb[i] = old + np.float32(1e-3)
        Lp, rp = _loss(p, kw, dy)
        sb[i] = old
        if all(np.array_equal(a, b_) for a, b_ in zip(rp, route0)):
            assert Lp == L0


def check_zero_and_linear(b=bwd):
    p, kw, dy = _problem(1)
    kw0 = dict(kw, aux_weight=0.0, z_weight=0.0)
    g0 = _grads(p, kw0, np.zeros_like(dy), b)
    for name in GRAD_OF.values():
        assert not np.any(getattr(g0, name)), name
    dy2 = np.random.default_rng(7).normal(size=dy.shape)
    ga, gb, gab = _grads(p, kw0, dy, b), _grads(p, kw0, dy2, b), _grads(p, kw0, dy + 2 * dy2, b)
    for name in GRAD_OF.values():
        np.testing.assert_allclose(getattr(gab, name), getattr(ga, name) + 2 * getattr(gb, name),
                                   rtol=1e-10, atol=1e-12)


def check_sparsity(b=bwd):
    # experts that no kept token chose get no gradient; dropped slots' weights neither
    p, kw, dy = _problem(2)
    g = _grads(p, kw, dy, b)
    fwd = orc.layer_forward(p["x"], p["w_router"], p["bias"], p["w1"], p["w3"], p["w2"], k=kw["k"],
                            cap=kw["cap"], bf16=False, align=kw["align"], tokens=[],
                            selection_bias=kw["selection_bias"])
    kept = fwd.disp.row_map >= 0
    assert np.any(~kept), "the pin needs a dropped slot"
    assert np.all(g.dweights[~kept] == 0)
    for e in range(p["w1"].shape[0]):
        if not np.any((fwd.idx == e) & kept):
            assert not np.any(g.dw1[e]) and not np.any(g.dw2[e])


def test_finite_differences():
    check_finite_differences()


def test_finite_differences_other_seed():
    check_finite_differences(seed=3)


def test_finite_differences_without_extras():
    p, kw, dy = _problem(4, shared=False, bias=False, selection=False)
    g = _grads(p, kw, dy)
    eps = 1e-6
    for name in ("x", "w_router", "w2"):
        flat = p[name].reshape(-1)
        c = 3
        old = flat[c]
        flat[c] = old + eps
        Lp, _ = _loss(p, kw, dy)
        flat[c] = old - eps
        Lm, _ = _loss(p, kw, dy)
        flat[c] = old
        assert abs((Lp - Lm) / (2 * eps) - getattr(g, GRAD_OF[name]).reshape(-1)[c]) < 1e-5
    assert g.dbias is None and g.dws1 is None


def test_zero_and_linear():
    check_zero_and_linear()


def test_sparsity():
    check_sparsity()


# --------------------------------------------------------------------------
# mutation tests
# --------------------------------------------------------------------------

def _mut_silu_grad_sigma_only(u):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-u))


_EXPERT_BWD = bwd.expert_backward


def _mut_expert_swap(x64, w1, w3, w2, dout):
    return _EXPERT_BWD(x64, w3, w1, w2, dout)


def _patched_backward(pattern, replacement):
    """layer_backward with one line of its arithmetic altered (a planted mistake)."""
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(bwd.layer_backward))
    assert pattern in src, pattern
    ns = dict(bwd.__dict__)
    exec(src.replace(pattern, replacement), ns)
    return ns["layer_backward"]


MUTANTS = [
    ("no_renorm_term", "(dwt - np.sum(dwt * w, axis=1, keepdims=True)) / S", "dwt / S"),
    ("aux_without_N", "aux_weight * N * f[None, :] / T", "aux_weight * f[None, :] / T"),
    ("z_without_2", "z_weight * (2.0 / T) * lse * s", "z_weight * (1.0 / T) * lse * s"),
    ("router_transposed", "dx += dg @ orc.as_f64(w_router).T", "dx += (dg @ orc.as_f64(w_router).T)[:, ::-1]"),
    ("dropped_weights_get_grad", "ti, tj = np.nonzero((idx == e) & kept)", "ti, tj = np.nonzero(idx == e)"),
    ("softmax_bwd_no_centering", "dg = s * (ds - np.sum(ds * s, axis=1, keepdims=True))", "dg = s * ds"),
]


@pytest.mark.parametrize("name,pattern,replacement", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, pattern, replacement, monkeypatch):
    monkeypatch.setattr(bwd, "layer_backward", _patched_backward(pattern, replacement))
    caught = []
    for chk in (check_finite_differences, check_zero_and_linear, check_sparsity):
        try:
            chk(bwd)
        except AssertionError:
            caught.append(chk.__name__)
    assert caught, name


@pytest.mark.parametrize("name,fn", [("silu_grad", _mut_silu_grad_sigma_only),
                                     ("expert_backward", _mut_expert_swap)])
def test_function_mutant_is_caught(name, fn, monkeypatch):
    monkeypatch.setattr(bwd, name, fn)
    with pytest.raises(AssertionError):
        check_finite_differences(bwd)
