"""Pins of the fp64 backward oracle (oracle/ipttt_backward.py).

The gradients are derived by hand, so each one is checked against something that
does not share that derivation:
  * central finite differences of the forward oracle, element by element, for every
    input and weight, on a tiny batch that has documents starting inside a chunk, on
    a chunk boundary and twice in one chunk, a ragged last chunk, a clip threshold
    that some chunks exceed and some do not, and a gradient on the final state;
  * with eta = 0 the layer is a plain gated MLP, whose gradients torch autograd
    gives in fp64, and the conv and target weights get no gradient at all.
"""
import numpy as np
import pytest
import torch

from oracle import ipttt_backward as bw
from oracle import ipttt_oracle as fw

B, T, C, d, F = 2, 13, 4, 3, 5
# row 0: a document starts inside chunk 1 (token 6); row 1: one on the chunk
# boundary at 8 and another at 10, both in chunk 2; the last chunk is one token
DOC_STARTS = [6, T + 8, T + 10]
NAMES = ("H", "X0", "Wgate", "Wup", "Wdown0", "conv_w", "Wtarget")


def make_inputs(seed):
    r = np.random.default_rng(seed)
    return {
        "H": r.standard_normal((B, T, d)),
        "X0": r.standard_normal((B, T, d)),
        "Wgate": r.standard_normal((F, d)) * 0.7,
        "Wup": r.standard_normal((F, d)) * 0.7,
        "Wdown0": r.standard_normal((d, F)) * 0.5,
        "conv_w": r.standard_normal((d, fw.CONV_TAPS)) * 0.6,
        "Wtarget": r.standard_normal((d, d)) * 0.6,
    }


def chunk_norms(p, eta):
    """||eta P_i|| of every chunk of every row, from the forward oracle's pieces."""
    flags = fw.start_flags(B, T, DOC_STARTS)
    out = []
    for b in range(B):
        Z = fw.gated_activation(p["H"][b], p["Wgate"], p["Wup"])
        V = fw.lm_target(p["X0"][b], p["conv_w"], p["Wtarget"], C, flags[b])
        for (s, e, f, l, cont, has_start) in fw.chunk_segments(flags[b], C):
            out.append(np.linalg.norm(fw.hebbian_delta(Z[l:e], V[l:e], eta)))
    return np.asarray(out)


def split_tau(norms):
    """A threshold between two middle norms, so that some chunks clip and some do not,
    and well away from every norm (the clip has a kink at ||eta P|| = tau)."""
    s = np.sort(norms)
    gaps = s[1:] / s[:-1]
    mid = len(s) // 2
    j = max(range(1, len(s) - 2), key=lambda i: gaps[i] - 0.1 * abs(i - mid))
    tau = float(np.sqrt(s[j] * s[j + 1]))
    assert np.min(np.abs(norms - tau)) / tau > 1e-2
    return tau


def probe_loss(p, eta, tau, gO, gS):
    """L = <gO, O> + <gS, S_final>: its gradient is the backward of (gO, gS)."""
    r = fw.layer_forward(p["H"], p["X0"], p["Wgate"], p["Wup"], p["Wdown0"], p["conv_w"],
                         p["Wtarget"], C, DOC_STARTS, eta, tau)
    L = float(np.sum(gO * r["O"]))
    if gS is not None:
        L += float(np.sum(gS * r["S_final"]))
    return L


def finite_difference(p, name, eta, tau, gO, gS, h=1e-5):
    g = np.zeros_like(p[name])
    for idx in np.ndindex(p[name].shape):
        q = {k: v.copy() for k, v in p.items()}
        q[name][idx] += h
        up = probe_loss(q, eta, tau, gO, gS)
        q[name][idx] -= 2 * h
        dn = probe_loss(q, eta, tau, gO, gS)
        g[idx] = (up - dn) / (2 * h)
    return g


def backward(p, eta, tau, gO, gS):
    return bw.layer_backward(p["H"], p["X0"], p["Wgate"], p["Wup"], p["Wdown0"], p["conv_w"],
                             p["Wtarget"], C, DOC_STARTS, eta, tau, gO, gS)


def assert_close(got, want, name):
    scale = max(np.max(np.abs(want)), 1e-12)
    err = np.max(np.abs(got - want)) / scale
    assert err < 1e-6, f"{name}: max error {err:.3e} of max |grad| {scale:.3e}"


def test_layout_of_the_pinned_case():
    # the case reaches every branch of the backward scan
    flags = fw.start_flags(B, T, DOC_STARTS)
    segs = [fw.chunk_segments(flags[b], C) for b in range(B)]
    kinds = [(cont, has_start, f < e, l > s) for row in segs for (s, e, f, l, cont, has_start) in row]
    assert any(c and h for c, h, _, _ in kinds)          # continues a document and starts one
    assert any(c and not h for c, h, _, _ in kinds)      # continues, no start: state carried
    assert any(not c for c, _, _, _ in kinds)            # begins on a document start
    assert segs[1][2][3] == 10                           # two starts: last segment from 10
    assert segs[0][-1][1] - segs[0][-1][0] == 1          # ragged one-token chunk


@pytest.mark.parametrize("clip", ["split", "none", "all"])
@pytest.mark.parametrize("final_grad", [False, True])
def test_backward_matches_finite_differences(clip, final_grad):
    p = make_inputs(11)
    eta = 0.3
    norms = chunk_norms(p, eta)
    tau = {"split": split_tau(norms), "none": 0.0, "all": 0.5 * float(np.min(norms))}[clip]
    if clip == "split":
        assert np.any(norms > tau) and np.any(norms < tau)
    r = np.random.default_rng(12)
    gO = r.standard_normal((B, T, d))
    gS = r.standard_normal((B, d, F)) if final_grad else None
    got = backward(p, eta, tau, gO, gS)
    for name in NAMES:
        assert_close(got[name], finite_difference(p, name, eta, tau, gO, gS), name)


def test_zero_learning_rate_is_the_plain_gated_mlp():
    p = make_inputs(21)
    gO = np.random.default_rng(22).standard_normal((B, T, d))
    got = backward(p, 0.0, 0.0, gO, None)
    t = {k: torch.tensor(p[k], dtype=torch.float64, requires_grad=True)
         for k in ("H", "Wgate", "Wup", "Wdown0")}
    Z = torch.nn.functional.silu(t["H"] @ t["Wgate"].T) * (t["H"] @ t["Wup"].T)
    O = Z @ t["Wdown0"].T
    O.backward(torch.tensor(gO))
    for name in ("H", "Wgate", "Wup", "Wdown0"):
        np.testing.assert_allclose(got[name], t[name].grad.numpy(), rtol=1e-12, atol=1e-12)
    for name in ("X0", "conv_w", "Wtarget"):
        assert not np.any(got[name])


def test_clipped_delta_gradient_is_orthogonal_to_the_delta():
    # with the clip active every delta has norm tau whatever the scale of P; V, and
    # so P, is linear in Wtarget, so when every chunk clips and only S_final is
    # probed, the loss does not change along Wtarget's own direction
    p = make_inputs(31)
    eta = 0.3
    tau = 0.25 * float(np.min(chunk_norms(p, eta)))
    gO = np.zeros((B, T, d))
    gS = np.random.default_rng(32).standard_normal((B, d, F))
    got = backward(p, eta, tau, gO, gS)
    assert abs(float(np.sum(p["Wtarget"] * got["Wtarget"]))) < 1e-10 * np.linalg.norm(got["Wtarget"]) * np.linalg.norm(p["Wtarget"])
    assert np.linalg.norm(got["Wtarget"]) > 1e-3
