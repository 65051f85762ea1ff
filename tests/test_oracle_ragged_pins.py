"""Pins of the oracle's ragged (variable-length) folding against what the pages and the
mathematics fix, not against the oracle itself:

* equal lengths reduce to the batched layer, bitwise (the fixed-period fold is the
  special case of the offsets);
* the definition (each sample on its own slice) equals the fold read literally -- one
  recurrence along the packed row with the transition forced to 0 at every offset and a
  conv that never reads across an offset -- written apart in numpy;
* a closed form per sample (constant inputs, N = 1): each sample's geometric sum restarts
  at its own offset, whatever the other samples' lengths;
* sample isolation: nan written into one sample leaves every other sample's outputs
  bitwise unchanged in the literal form, which runs straight through the boundaries.

Passages: the fold with Abar_t = 0 at each sample start (sungsoo.github.io section 3.3
equations; techloop.online, Batch Folding with Periodic State Reset) and the conv that
must not cross folded sample boundaries (techloop.online, convolution-boundary paragraph),
with the fixed period replaced by per-sample offsets."""
import numpy as np
import pytest

import oracle


def _inputs(D, N, lens, aux, seed):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    Lt, S = int(cu[-1]), len(lens)
    Lx = Lt - 2 * S if aux else Lt
    return dict(x=rng.standard_normal((D, Lx)), dt=0.5 * rng.standard_normal((D, Lt)), z=rng.standard_normal((D, Lt)),
                Bm=rng.standard_normal((N, Lt)), Cm=rng.standard_normal((N, Lt)),
                A=-np.exp(rng.standard_normal((D, N))), Dskip=rng.standard_normal(D),
                dt_bias=np.log(np.expm1(rng.uniform(1e-3, 1e-1, D))), conv_w=rng.uniform(-0.5, 0.5, (D, 4)),
                conv_b=rng.uniform(-0.5, 0.5, D)), cu


def _call(f, d, cu, **kw):
    return f(d["x"], d["dt"], d["z"], d["Bm"], d["Cm"], d["A"], d["Dskip"], d["dt_bias"], d["conv_w"], d["conv_b"],
             cu, **kw)


@pytest.mark.parametrize("aux,swap", [(False, False), (True, True), (True, False)])
def test_equal_lengths_are_the_batched_layer(aux, swap):
    S, D, N, L = 4, 6, 5, 9
    d, cu = _inputs(D, N, [L] * S, aux, seed=1)
    y = _call(oracle.mixer_layer_varlen, d, cu, aux_init_in=aux, swap_out=swap)
    T = L - 2 if aux else L
    xb = d["x"].reshape(D, S, T).transpose(1, 0, 2)
    pk = lambda a: a.reshape(a.shape[0], S, L).transpose(1, 0, 2)
    yb = oracle.mixer_layer(xb, pk(d["dt"]), pk(d["z"]), pk(d["Bm"]), pk(d["Cm"]), d["A"], d["Dskip"], d["dt_bias"],
                            d["conv_w"], d["conv_b"], aux_init_in=aux, swap_out=swap)
    assert np.array_equal(y, yb.transpose(1, 0, 2).reshape(D, S * L))


@pytest.mark.parametrize("aux,swap,pad_left,lens", [
    (False, False, 1, [7, 3, 12, 5]),
    (False, True, 3, [1, 0, 9, 2, 0, 4]),   # empty samples and a one-token sample
    (True, True, 1, [3, 11, 5, 8]),         # the shortest aux sample: one patch token
    (True, False, 0, [20, 4, 6]),
])
def test_definition_equals_literal_packed_fold(aux, swap, pad_left, lens):
    d, cu = _inputs(6, 4, lens, aux, seed=2)
    y1 = _call(oracle.mixer_layer_varlen, d, cu, aux_init_in=aux, swap_out=swap, pad_left=pad_left)
    y2 = _call(oracle.mixer_layer_packed_literal, d, cu, aux_init_in=aux, swap_out=swap, pad_left=pad_left)
    assert np.max(np.abs(y1 - y2)) <= 1e-12 * max(1.0, np.max(np.abs(y1)))


def test_closed_form_per_sample():
    """N = 1, no conv, no gate, constant u, Delta, B, C: in sample s at within-sample index
    t, h_t = Delta B u (1 - a^(t+1)) / (1 - a) with a = exp(Delta A), y_t = C h_t + Dskip u."""
    lens = [5, 1, 9, 3]
    cu = np.concatenate([[0], np.cumsum(lens)])
    Lt, D = int(cu[-1]), 2
    u0, delta, b0, c0, A0, dsk = 0.7, 0.3, 1.3, -0.8, -0.9, 0.25
    x = np.full((D, Lt), u0)
    dt = np.full((D, Lt), delta)
    Bm, Cm = np.full((1, Lt), b0), np.full((1, Lt), c0)
    A = np.full((D, 1), A0)
    y = oracle.mixer_layer_varlen(x, dt, None, Bm, Cm, A, np.full(D, dsk), None, None, None, cu, dt_softplus=False)
    a = np.exp(delta * A0)
    for s, L in enumerate(lens):
        t = np.arange(L)
        want = c0 * delta * b0 * u0 * (1 - a ** (t + 1)) / (1 - a) + dsk * u0
        np.testing.assert_allclose(y[:, cu[s]:cu[s + 1]], np.broadcast_to(want, (D, L)), rtol=1e-13, atol=0)


@pytest.mark.parametrize("aux", [False, True])
def test_isolation_in_the_literal_fold(aux):
    lens = [6, 9, 4, 7]
    d, cu = _inputs(5, 4, lens, aux, seed=3)
    kw = dict(aux_init_in=aux, swap_out=aux)
    y0 = _call(oracle.mixer_layer_packed_literal, d, cu, **kw)
    j = 1
    a, e = int(cu[j]), int(cu[j + 1])
    d2 = {k: v.copy() for k, v in d.items()}
    for k in ("dt", "z"):
        d2[k][:, a:e] = np.nan
    d2["Bm"][:, a:e] = np.inf
    xa, xe = (a - 2 * j, e - 2 * j - 2) if aux else (a, e)
    d2["x"][:, xa:xe] = np.nan
    y1 = _call(oracle.mixer_layer_packed_literal, d2, cu, **kw)
    keep = np.ones(int(cu[-1]), bool)
    keep[a:e] = False
    assert np.array_equal(y1[:, keep], y0[:, keep])
    assert np.isnan(y1[:, a:e]).all()


def test_final_states_are_the_per_sample_states():
    lens = [5, 0, 8]
    d, cu = _inputs(4, 3, lens, False, seed=4)
    y, fs = _call(oracle.mixer_layer_varlen, d, cu, want_state=True)
    for s, (a, e) in enumerate(zip(cu[:-1], cu[1:])):
        if e == a:
            assert not fs[s].any()
            continue
        _, f1 = oracle.mixer_layer(d["x"][None, :, a:e], d["dt"][None, :, a:e], d["z"][None, :, a:e],
                                   d["Bm"][None, :, a:e], d["Cm"][None, :, a:e], d["A"], d["Dskip"], d["dt_bias"],
                                   d["conv_w"], d["conv_b"], want_state=True)
        assert np.array_equal(fs[s], f1[0])
