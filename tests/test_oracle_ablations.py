"""Pins of the ablation oracle (oracle/ipttt_ablations.py), each against a fact that
does not come from the oracle's own code: a scalar case worked by hand, closed
forms and special cases, invariants, and agreement of two formulations."""
import numpy as np
import pytest

from oracle import ipttt_ablations as ab
from oracle import ipttt_oracle as fw


def scalar_row(z, v, w0, flags, eta, tau, form="direct"):
    Z = np.asarray(z, float)[:, None]
    V = np.asarray(v, float)[:, None]
    W0 = np.array([[w0]], float)
    return ab.FORMS[form](Z, V, W0, 1, np.asarray(flags, bool), eta, tau)


@pytest.mark.parametrize("form", list(ab.FORMS))
def test_scalar_case_worked_by_hand(form):
    # d = F = 1, one-token chunks, eta = 1, tau = 1, W0 = 0, z = 1 throughout, v = 2, 0.5, -3.
    #   chunk 0 (row start): O = 0; S + dW = 0 + 2 = 2 > 1, scale 1/2, S_1 = 1
    #   chunk 1: O = z S_1 = 1;   S_1 + dW = 1 + 0.5 = 1.5, scale 2/3, S_2 = 1
    #   chunk 2: O = z S_2 = 1;   S_2 + dW = 1 - 3 = -2,    scale 1/2, S_3 = -1
    O, D, S, c = scalar_row([1, 1, 1], [2, 0.5, -3], 0.0, [1, 0, 0], 1.0, 1.0, form)
    np.testing.assert_allclose(O[:, 0], [0.0, 1.0, 1.0], atol=1e-15)
    np.testing.assert_allclose(S, [[-1.0]], atol=1e-15)
    np.testing.assert_allclose(c, [0.5, 2.0 / 3.0, 0.5], atol=1e-15)
    # clipping each delta instead gives S_2 = 1 + 0.5 = 1.5, so O_2 = 1.5: the two
    # readings differ on this input
    O_delta, _, S_delta, _ = fw.core_sequential(np.ones((3, 1)), np.array([[2.0], [0.5], [-3.0]]),
                                                np.zeros((1, 1)), 1, np.array([1, 0, 0], bool), 1.0, 1.0)
    assert O_delta[2, 0] == 1.5 and S_delta[0, 0] == 0.5
    # a document starting at token 2: chunk 2 sees no state and restarts it
    #   chunk 2: O = 0;  S + dW = 0 - 3 = -3, scale 1/3, S_3 = -1
    O, D, S, c = scalar_row([1, 1, 1], [2, 0.5, -3], 0.0, [1, 0, 1], 1.0, 1.0, form)
    np.testing.assert_allclose(O[:, 0], [0.0, 1.0, 0.0], atol=1e-15)
    np.testing.assert_allclose(c, [0.5, 2.0 / 3.0, 1.0 / 3.0], atol=1e-15)
    np.testing.assert_allclose(S, [[-1.0]], atol=1e-15)


def draw(seed, B=2, T=23, d=4, F=6):
    r = np.random.default_rng(seed)
    return {"H": r.standard_normal((B, T, d)), "X0": r.standard_normal((B, T, d)),
            "Wgate": r.standard_normal((F, d)) * 0.6, "Wup": r.standard_normal((F, d)) * 0.6,
            "Wdown0": r.standard_normal((d, F)) * 0.4, "conv_w": r.standard_normal((d, 5)) * 0.5,
            "Wtarget": r.standard_normal((d, d)) * 0.5}


def run(p, C, docs, eta, tau, form="direct"):
    return ab.layer_forward_state_clip(p["H"], p["X0"], p["Wgate"], p["Wup"], p["Wdown0"], p["conv_w"],
                                       p["Wtarget"], C, docs, eta, tau, form)


def forward(p, C, docs, eta, tau):
    return fw.layer_forward(p["H"], p["X0"], p["Wgate"], p["Wup"], p["Wdown0"], p["conv_w"], p["Wtarget"], C,
                            docs, eta, tau)


DOCS = [9, 23 + 4, 23 + 12]


@pytest.mark.parametrize("form", list(ab.FORMS))
def test_no_clip_is_the_unclipped_forward(form):
    p = draw(1)
    for tau in (0.0, np.inf):
        got = run(p, 4, DOCS, 0.2, tau, form)
        ref = forward(p, 4, DOCS, 0.2, 0.0)
        np.testing.assert_allclose(got["O"], ref["O"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got["S_final"], ref["S_final"], rtol=1e-12, atol=1e-12)
        assert np.all(got["scale"] == 1.0)


@pytest.mark.parametrize("form", list(ab.FORMS))
def test_state_norm_never_exceeds_tau(form):
    p = draw(2)
    eta, C = 0.2, 4
    ref = forward(p, C, DOCS, eta, 0.0)
    tau = 0.3 * float(np.max(np.linalg.norm(ref["S_final"], axis=(1, 2))))
    got_any_clip = False
    for T_end in range(C, 23 + 1, C):
        q = dict(p, H=p["H"][:, :T_end], X0=p["X0"][:, :T_end])
        docs = [b * T_end + t for g in DOCS for b, t in [divmod(g, 23)] if t < T_end]
        r = run(q, C, docs, eta, tau, form)
        assert np.all(np.linalg.norm(r["S_final"], axis=(1, 2)) <= tau * (1 + 1e-12))
        got_any_clip |= bool(np.any(r["scale"] < 1.0))
    assert got_any_clip


def test_tiny_tau_holds_the_state_on_the_sphere():
    # when every accumulated state exceeds tau, each clip lands exactly on norm tau
    p = draw(3)
    tau = 1e-9
    r = run(p, 4, [], 0.2, tau)
    assert np.all(r["scale"] < 1.0)
    np.testing.assert_allclose(np.linalg.norm(r["S_final"], axis=(1, 2)), tau, rtol=1e-12)


def test_documents_of_one_chunk_match_the_delta_clip():
    # every chunk starts a document: the state before each delta is zero, so
    # clipping the state is clipping the delta
    p = draw(4, T=16)
    C = 4
    docs = [b * 16 + t for b in range(2) for t in range(C, 16, C)]
    ref = forward(p, C, docs, 0.3, 0.05)
    got = run(p, C, docs, 0.3, 0.05)
    assert np.any(ref["alpha"] < 1.0)
    np.testing.assert_allclose(got["scale"], ref["alpha"], rtol=1e-12)
    np.testing.assert_allclose(got["S_final"], ref["S_final"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(got["O"], ref["O"], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("C", [1, 3, 4, 7, 23])
def test_two_formulations_agree(C):
    p = draw(5)
    ref = forward(p, C, DOCS, 0.25, 0.0)
    tau = 0.5 * float(np.median(np.linalg.norm(ref["S_final"], axis=(1, 2))))
    a = run(p, C, DOCS, 0.25, tau, "direct")
    b = run(p, C, DOCS, 0.25, tau, "scaled")
    for k in ("O", "D", "S_final", "scale"):
        np.testing.assert_allclose(a[k], b[k], rtol=1e-10, atol=1e-12)


def test_causality():
    p = draw(6)
    C, eta = 4, 0.2
    tau = 0.5
    base = run(p, C, DOCS, eta, tau)
    for t in (0, 5, 11, 22):
        q = {k: v.copy() for k, v in p.items()}
        q["H"][:, t + 1:] += 1.0
        q["X0"][:, t + 1:] -= 1.0
        # only tokens of chunks after t's chunk may change: the conv looks ahead
        # inside the chunk, and the update reaches later chunks only
        end = (t // C) * C
        r = run(q, C, DOCS, eta, tau)
        np.testing.assert_array_equal(r["O"][:, :end], base["O"][:, :end])


def test_target_without_conv_is_the_projected_token():
    # tap 0 alone is never masked: V = X0 Wtarget exactly, at every chunk and document edge
    r = np.random.default_rng(7)
    X0 = r.standard_normal((19, 5))
    Wt = r.standard_normal((5, 5))
    flags = np.zeros(19, bool)
    flags[[0, 6, 13]] = True
    V = fw.lm_target(X0, ab.conv_without_lookahead(5), Wt, 4, flags)
    np.testing.assert_array_equal(V, X0 @ Wt)


def test_target_without_projection_is_the_conv():
    r = np.random.default_rng(8)
    X0 = r.standard_normal((19, 5))
    cw = r.standard_normal((5, 5))
    flags = np.zeros(19, bool)
    flags[[0, 6, 13]] = True
    np.testing.assert_array_equal(fw.lm_target(X0, cw, ab.target_without_projection(5), 4, flags),
                                  fw.conv_target_input(X0, cw, 4, flags))
