"""Pins of the fp64 oracle to facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute the same way:
hand-worked values, a library routine (torch's SiLU, linear, depthwise conv1d),
a finite-difference gradient, the other two formulations of the scan, the
induction-head closed form, or an invariance (causality, document reset).
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import ipttt_oracle as orc

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")
FORMS = ("sequential", "prefix_sum", "bruteforce")


def rnd(seed, *shape, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def small_layer(seed, B=1, T=24, d=6, F=10, C=5):
    H = rnd(seed, B, T, d)
    X0 = rnd(seed + 1, B, T, d)
    Wg = rnd(seed + 2, F, d, scale=d ** -0.5)
    Wu = rnd(seed + 3, F, d, scale=d ** -0.5)
    W0 = rnd(seed + 4, d, F, scale=F ** -0.5)
    cw = rnd(seed + 5, d, 5, scale=0.3)
    Wt = np.eye(d) + rnd(seed + 6, d, d, scale=0.1)
    return H, X0, Wg, Wu, W0, cw, Wt


# --- hand-worked values -------------------------------------------------------

@pytest.mark.parametrize("form", FORMS)
def test_hand_worked_cases(form):
    for case in json.load(open(GOLD))["cases"]:
        Z = np.asarray(case["Z"], float)[None]
        V = np.asarray(case["V"], float)[None]
        W0 = np.asarray(case["W0"], float)
        r = orc.core_forward(Z, V, W0, case["C"], case["doc_starts"], case["eta"], case["tau"], form)
        for key in ("O", "D", "S_final", "alpha"):
            np.testing.assert_allclose(r[key][0], np.asarray(case[key], float), rtol=0, atol=1e-12,
                                       err_msg=f"{case['name']} {key} ({form})")


def test_hand_worked_conv():
    for case in json.load(open(GOLD))["conv_cases"]:
        X0 = np.asarray(case["X0"], float)
        T = X0.shape[0]
        flags = orc.start_flags(1, T, case["doc_starts"])[0]
        U = orc.conv_target_input(X0, np.asarray(case["conv_w"], float), case["C"], flags)
        np.testing.assert_allclose(U, np.asarray(case["U"], float), atol=0)
        V = orc.lm_target(X0, np.asarray(case["conv_w"], float), np.asarray(case["Wtarget"], float),
                          case["C"], flags)
        np.testing.assert_allclose(V, np.asarray(case["V"], float), atol=0)


# --- library routines ---------------------------------------------------------

def torch_gated_mlp(H, Wg, Wu, W0):
    h = torch.from_numpy(H)
    z = torch.nn.functional.silu(torch.nn.functional.linear(h, torch.from_numpy(Wg)))
    z = z * torch.nn.functional.linear(h, torch.from_numpy(Wu))
    return torch.nn.functional.linear(z, torch.from_numpy(W0)).numpy(), z.numpy()


def test_eta_zero_is_plain_gated_mlp():
    H, X0, Wg, Wu, W0, cw, Wt = small_layer(1, B=2, T=30, C=4)
    r = orc.layer_forward(H, X0, Wg, Wu, W0, cw, Wt, 4, [37], 0.0, 0.0)
    ref, zref = torch_gated_mlp(H, Wg, Wu, W0)
    np.testing.assert_allclose(r["O"], ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["Z"], zref, rtol=1e-12, atol=1e-12)
    assert np.all(r["D"] == 0)


def test_zero_conv_is_plain_gated_mlp():
    """Zero-initialised conv (the paper's init) makes the target, hence every delta, zero."""
    H, X0, Wg, Wu, W0, cw, Wt = small_layer(2, T=40, C=8)
    r = orc.layer_forward(H, X0, Wg, Wu, W0, np.zeros_like(cw), Wt, 8, [], 0.5, 0.0)
    ref, _ = torch_gated_mlp(H, Wg, Wu, W0)
    np.testing.assert_allclose(r["O"], ref, rtol=1e-12, atol=1e-12)


def torch_segmented_conv(X0, cw, C, flags):
    """Depthwise conv1d (torch) run separately on every chunk/document piece, right-padded."""
    T, d = X0.shape
    cut = sorted(set(list(range(0, T, C)) + [t for t in range(T) if flags[t]] + [T]))
    out = np.zeros((T, d))
    w = torch.from_numpy(cw).unsqueeze(1)  # [d, 1, 5]
    for a, b in zip(cut[:-1], cut[1:]):
        x = torch.from_numpy(X0[a:b].T.copy()).unsqueeze(0)  # [1, d, L]
        x = torch.nn.functional.pad(x, (0, 4))
        out[a:b] = torch.nn.functional.conv1d(x, w, groups=d)[0].T.numpy()
    return out


@pytest.mark.parametrize("C,starts", [(8, []), (5, [3, 11, 12, 30]), (1, [7])])
def test_conv_matches_torch_depthwise_conv1d(C, starts):
    _, X0, _, _, _, cw, _ = small_layer(3, T=40)
    flags = orc.start_flags(1, 40, starts)[0]
    U = orc.conv_target_input(X0[0], cw, C, flags)
    np.testing.assert_allclose(U, torch_segmented_conv(X0[0], cw, C, flags), rtol=1e-12, atol=1e-12)


# --- calculus / closed forms ----------------------------------------------------

def test_update_is_negative_gradient_of_inner_product_loss():
    """dW = -eta grad_W L with L(W) = -<Z W^T, V>_F, by central differences."""
    Z, V, W = rnd(4, 7, 5), rnd(5, 7, 3), rnd(6, 3, 5)
    eta = 0.37

    def loss(Wm):
        return -float(np.sum((Z @ Wm.T) * V))

    g = np.zeros_like(W)
    h = 1e-6
    for i in range(W.shape[0]):
        for j in range(W.shape[1]):
            e = np.zeros_like(W)
            e[i, j] = h
            g[i, j] = (loss(W + e) - loss(W - e)) / (2 * h)
    np.testing.assert_allclose(orc.hebbian_delta(Z, V, eta), -eta * g, rtol=1e-7, atol=1e-8)


def test_clip_scales_to_threshold():
    Z, V = rnd(7, 6, 9), rnd(8, 6, 4)
    dW = orc.hebbian_delta(Z, V, 1.0)
    n = np.linalg.norm(dW)
    a = orc.clip_factor(n, n / 3)
    assert abs(np.linalg.norm(a * dW) - n / 3) < 1e-12 * n
    assert orc.clip_factor(n, 2 * n) == 1.0
    assert orc.clip_factor(n, 0.0) == 1.0 and orc.clip_factor(n, float("inf")) == 1.0


def test_single_chunk_uses_w0_only():
    H, X0, Wg, Wu, W0, cw, Wt = small_layer(9, T=16, C=16)
    r = orc.layer_forward(H, X0, Wg, Wu, W0, cw, Wt, 16, [], 0.3, 0.0)
    ref, _ = torch_gated_mlp(H, Wg, Wu, W0)
    np.testing.assert_allclose(r["O"], ref, rtol=1e-12, atol=1e-12)
    assert np.any(r["S_final"] != 0)


def theorem_setup(target):
    """Induction-head case: keys/values are one-hot embeddings (epsilon = 0)."""
    d, F, C, T = 8, 6, 4, 8
    Z = np.zeros((1, T, F))
    V = np.zeros((1, T, d))
    W0 = np.zeros((d, F))
    t_star, n, k_star, v_star = 1, 6, 2, 5
    z = np.zeros(F); z[3] = 1.0
    Z[0, t_star] = z
    Z[0, n] = z
    for t in range(T):
        if t not in (t_star, n):
            Z[0, t, t % 3] = 0.7          # orthogonal to z_n
            V[0, t, (t + 1) % d] = 1.0
    V[0, t_star] = np.eye(d)[v_star if target == "lm" else k_star]
    return Z, V, W0, C, n, v_star


@pytest.mark.parametrize("form", FORMS)
def test_theorem1_lm_target_raises_the_right_logit(form):
    eta = 0.25
    Z, V, W0, C, n, v_star = theorem_setup("lm")
    r = orc.core_forward(Z, V, W0, C, [], eta, 0.0, form)
    expect = np.zeros(V.shape[2]); expect[v_star] = eta
    np.testing.assert_allclose(r["O"][0, n], expect, atol=1e-15)


@pytest.mark.parametrize("form", FORMS)
def test_theorem1_reconstruction_target_leaves_it(form):
    Z, V, W0, C, n, v_star = theorem_setup("reconstruction")
    r = orc.core_forward(Z, V, W0, C, [], 0.25, 0.0, form)
    assert r["O"][0, n, v_star] == 0.0


def test_lm_target_through_the_conv_is_next_token():
    """Taps [0,1,0,0,0] with Wtarget = I give V_t = X0_{t+1} inside a chunk, 0 at its end."""
    T, d, C = 12, 5, 4
    X0 = rnd(10, T, d)
    cw = np.zeros((d, 5)); cw[:, 1] = 1.0
    V = orc.lm_target(X0, cw, np.eye(d), C, orc.start_flags(1, T, [])[0])
    for t in range(T):
        want = X0[t + 1] if (t + 1) % C != 0 else np.zeros(d)
        np.testing.assert_array_equal(V[t], want)
    cw = np.zeros((d, 5)); cw[:, 0] = 1.0      # reconstruction target
    np.testing.assert_array_equal(orc.lm_target(X0, cw, np.eye(d), C, orc.start_flags(1, T, [])[0]), X0)


# --- three formulations and invariances ------------------------------------------

@pytest.mark.parametrize("C", [1, 2, 3, 5, 24])
@pytest.mark.parametrize("clip", [0.0, 0.05])
def test_three_formulations_agree(C, clip):
    H, X0, Wg, Wu, W0, cw, Wt = small_layer(11 + C, B=2, T=24, d=8, F=16)
    starts = [5, 6, 17, 24 + 9, 24 + 10, 24 + 22]
    res = [orc.layer_forward(H, X0, Wg, Wu, W0, cw, Wt, C, starts, 0.2, clip, f) for f in FORMS]
    for r in res[1:]:
        for key in ("O", "D", "S_final", "alpha"):
            np.testing.assert_allclose(r[key], res[0][key], rtol=1e-10, atol=1e-12, err_msg=key)
    if clip > 0:
        assert np.any(res[0]["alpha"] < 1.0)


def test_causality_every_token():
    """Perturbing any token s changes no output row t < s, within chunk(s) included."""
    H, X0, Wg, Wu, W0, cw, Wt = small_layer(20, T=20, C=5)
    base = orc.layer_forward(H, X0, Wg, Wu, W0, cw, Wt, 5, [13], 0.4, 0.0)["O"]
    for s in (3, 7, 12, 19):
        H2, X2 = H.copy(), X0.copy()
        H2[:, s:] += 1.0
        X2[:, s:] -= 2.0
        o = orc.layer_forward(H2, X2, Wg, Wu, W0, cw, Wt, 5, [13], 0.4, 0.0)["O"]
        np.testing.assert_array_equal(o[:, :s], base[:, :s])
        assert np.any(o[:, s:] != base[:, s:])


def test_prefix_oracle_reproduces_prefix():
    H, X0, Wg, Wu, W0, cw, Wt = small_layer(21, T=30, C=6)
    full = orc.layer_forward(H, X0, Wg, Wu, W0, cw, Wt, 6, [8], 0.4, 0.05)
    pre = orc.layer_forward(H[:, :12], X0[:, :12], Wg, Wu, W0, cw, Wt, 6, [8], 0.4, 0.05)
    np.testing.assert_array_equal(pre["O"], full["O"][:, :12])
    np.testing.assert_array_equal(pre["alpha"], full["alpha"][:, :2])


def test_chunk_aligned_documents_equal_separate_runs():
    H, X0, Wg, Wu, W0, cw, Wt = small_layer(22, T=24, C=4)
    packed = orc.layer_forward(H, X0, Wg, Wu, W0, cw, Wt, 4, [8, 20], 0.3, 0.0)
    for a, b in ((0, 8), (8, 20), (20, 24)):
        sep = orc.layer_forward(H[:, a:b], X0[:, a:b], Wg, Wu, W0, cw, Wt, 4, [], 0.3, 0.0)
        np.testing.assert_allclose(packed["O"][:, a:b], sep["O"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(packed["S_final"], sep["S_final"], rtol=1e-13, atol=1e-15)


def test_document_isolation_unaligned():
    """Changing document A's tokens never changes document B's outputs."""
    H, X0, Wg, Wu, W0, cw, Wt = small_layer(23, T=30, C=7)
    starts = [9, 17]
    base = orc.layer_forward(H, X0, Wg, Wu, W0, cw, Wt, 7, starts, 0.3, 0.0)["O"]
    H2, X2 = H.copy(), X0.copy()
    H2[:, 9:17] *= -1.5
    X2[:, 9:17] += 3.0
    o = orc.layer_forward(H2, X2, Wg, Wu, W0, cw, Wt, 7, starts, 0.3, 0.0)["O"]
    np.testing.assert_array_equal(o[:, :9], base[:, :9])
    np.testing.assert_array_equal(o[:, 17:], base[:, 17:])
    assert np.any(o[:, 9:17] != base[:, 9:17])


def test_hand_worked_stack():
    """stack_forward against a two-layer residual chain worked by hand."""
    for case in json.load(open(GOLD))["stack_cases"]:
        layers = [{k: np.asarray(v, float) for k, v in l.items()} for l in case["layers"]]
        H0 = np.asarray(case["H0"], float)[None]
        X0 = np.asarray(case["X0"], float)[None]
        Hout, outs = orc.stack_forward(layers, X0, H0, case["C"], case["doc_starts"], case["eta"], case["tau"])
        np.testing.assert_allclose(Hout[0], np.asarray(case["H_out"], float), rtol=1e-13, atol=1e-13)
        for l, r in enumerate(outs):
            np.testing.assert_allclose(r["O"][0], np.asarray(case["O"][l], float), rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(r["S_final"][0], np.asarray(case["S_final"][l], float), rtol=1e-13,
                                       atol=1e-13)


def test_stack_residual():
    H, X0, Wg, Wu, W0, cw, Wt = small_layer(24, T=12, C=4)
    p = dict(Wgate=Wg, Wup=Wu, Wdown0=W0, conv_w=cw, Wtarget=Wt)
    Hout, outs = orc.stack_forward([p, p], X0, H, 4, [], 0.2, 0.0)
    r0 = orc.layer_forward(H, X0, Wg, Wu, W0, cw, Wt, 4, [], 0.2, 0.0)
    r1 = orc.layer_forward(H + r0["O"], X0, Wg, Wu, W0, cw, Wt, 4, [], 0.2, 0.0)
    np.testing.assert_array_equal(Hout, H + r0["O"] + r1["O"])
    np.testing.assert_array_equal(outs[1]["O"], r1["O"])
