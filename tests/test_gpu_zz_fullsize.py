"""Parity at the full sizes of the layer's headline workloads, run in the same
launch configuration the benchmark times.  Collected after the small-shape parity
tests, so a failure here never hides them.

Checks against the fp64 oracle:
  * prefix: outputs depend only on earlier tokens (apply before update, conv looks
    at most to the chunk end), so the oracle run on the first chunks of a row
    reproduces the GPU outputs on those chunks (O, D, alpha);
  * the whole state walk: the oracle's chunk-by-chunk scan of a row
    (tests/fullsize_ref.py) gives every chunk's alpha, the final state S_final and
    the state a late chunk is applied with, hence that chunk's fast-weight term D;
    S_final and D are held to the bf16 bars, and S_final to carry no scale bias;
  * late output rows: O[t] = z_t W0^T + D[t] with |D[t]| <= |z_t| * sum_i alpha_i
    ||dW_i||_F <= |z_t| k tau, so sampled rows of the last chunk must lie within the
    bf16 tolerance plus that bound of the oracle's z_t W0^T.
"""
import gc

import numpy as np
import pytest
import torch

from chunk_wise_weight_gate_b200 import ipttt as ip
from chunk_wise_weight_gate_b200 import synth
from oracle import ipttt_oracle as orc
from tests import fullsize_ref
from tests.gpu_util import BIAS_TOL, WEIGHTS, maxrel, normrel, scale_bias

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

TOL_O = 2e-2
PREFIX_CHUNKS = 2
_STACK_INPUTS = {}


def stack_inputs(w, layer):
    """Per-layer inputs of the stack workload; they do not depend on the chunk size."""
    key = (layer,)
    if key not in _STACK_INPUTS:
        _STACK_INPUTS[key] = synth.make_inputs(w, seed=0, layer=layer, with_activations=(layer == 0))
    return _STACK_INPUTS[key]


def f64(t):
    return t.detach().double().cpu().numpy()


def row_docs(docs, b, T, lo, hi):
    """doc_starts of row b inside [lo, hi), shifted to the window (row start implicit)."""
    g = np.asarray(docs, dtype=np.int64)
    sel = g[(g // T == b) & (g % T >= lo) & (g % T < hi)] % T - lo
    return sel[sel > 0]


def oracle_window(inp, w, b, lo, hi, weights=None):
    wt = weights or {k: inp[k].double().numpy() for k in WEIGHTS}
    H = inp["H"][b:b + 1, lo:hi].double().numpy()
    X0 = inp["X0"][b:b + 1, lo:hi].double().numpy()
    return orc.layer_forward(H, X0, wt["Wgate"], wt["Wup"], wt["Wdown0"], wt["conv_w"], wt["Wtarget"], w.C,
                             row_docs(inp["doc_starts"].numpy(), b, w.T, lo, hi), w.eta, w.clip)


def run_layer(w, inp, debug=("D", "alpha")):
    dev = torch.device("cuda")
    cfg = ip.LayerConfig(B=w.B, T=w.T, d=w.d, F=w.F, C=w.C, eta=w.eta, clip=w.clip)
    t = {k: inp[k].to(dev) for k in ("H", "X0") + WEIGHTS}
    out = ip.forward(cfg, *(t[k] for k in ("H", "X0") + WEIGHTS), inp["doc_starts"], debug=debug)
    torch.cuda.synchronize()
    assert ip.get_status() == 0
    res = {k: v.cpu() for k, v in out.items() if v is not None}
    del t, out
    gc.collect()
    torch.cuda.empty_cache()
    return res


def check_prefix(out, inp, w, rows):
    n = PREFIX_CHUNKS * w.C
    for b in rows:
        ref = oracle_window(inp, w, b, 0, n)
        assert maxrel(f64(out["O"][b, :n]), ref["O"][0]) <= TOL_O
        np.testing.assert_allclose(f64(out["alpha"][b, :PREFIX_CHUNKS]), ref["alpha"][0], rtol=1e-2)
        if np.any(ref["D"] != 0):
            assert normrel(f64(out["D"][b, :n]), ref["D"][0]) <= 2e-2
            assert maxrel(f64(out["D"][b, :n]), ref["D"][0]) <= 5e-2


def check_late_chunks(out, inp, w, b, chunks):
    wt = {k: inp[k].double().numpy() for k in WEIGHTS}
    for c in chunks:
        lo, hi = c * w.C, min((c + 1) * w.C, w.T)
        ref = oracle_window(inp, w, b, lo, hi, wt)
        np.testing.assert_allclose(float(out["alpha"][b, c]), ref["alpha"][0, 0], rtol=1e-2)
    # sampled output rows of the last chunk
    k = (w.T + w.C - 1) // w.C
    t_rows = np.linspace((k - 1) * w.C, w.T - 1, 6).astype(int)
    H = inp["H"][b, t_rows].double().numpy()
    z = orc.gated_activation(H, wt["Wgate"], wt["Wup"])
    base = z @ wt["Wdown0"].T
    tau = w.clip if w.clip > 0 else np.inf
    bound = np.linalg.norm(z, axis=1, keepdims=True) * k * tau
    err = np.abs(f64(out["O"][b, t_rows]) - base)
    scale = np.max(np.abs(base))
    assert np.all(err <= TOL_O * scale + bound), float(np.max(err - bound))


def check_state_walk(out, w, name, b):
    """S_final, every alpha and the last chunk's D of row b against the oracle's scan."""
    k = (w.T + w.C - 1) // w.C
    late = k - 1
    S_ref, a_ref, states = fullsize_ref.scan_row(name, b, (late,))
    np.testing.assert_allclose(f64(out["alpha"][b]), a_ref, rtol=1e-2)
    S = f64(out["S_final"][b])
    _, D_ref = states[late]
    D = f64(out["D"][b, late * w.C:min(k * w.C, w.T)])
    print(f"{name} row {b}: S_final normrel {normrel(S, S_ref):.3e}, scale bias {scale_bias(S, S_ref):+.3e}; "
          f"chunk {late} D normrel {normrel(D, D_ref):.3e} maxrel {maxrel(D, D_ref):.3e}")
    assert normrel(S, S_ref) <= 2e-2
    assert abs(scale_bias(S, S_ref)) <= BIAS_TOL
    if np.any(D_ref != 0):
        assert normrel(D, D_ref) <= 2e-2
        assert maxrel(D, D_ref) <= 5e-2
    else:
        assert np.all(D == 0)


@pytest.mark.parametrize("name", ["qwen3_4b_32k", "qwen3_4b_128k", "packed_8x8k"])
def test_full_size_layer(name):
    w = synth.WORKLOADS[name]
    inp = fullsize_ref.inputs(name)
    out = run_layer(w, inp, debug=("D", "alpha", "S_final"))
    assert torch.isfinite(out["O"].float()).all()
    rows = list(range(w.B)) if w.B <= 2 else [0, w.B // 2, w.B - 1]
    check_prefix(out, inp, w, rows)
    k = (w.T + w.C - 1) // w.C
    check_late_chunks(out, inp, w, rows[-1], [k // 2, k - 1])
    for b in (rows[0], rows[-1]) if len(rows) > 1 else rows:
        check_state_walk(out, w, name, b)
    if w.clip > 0 and w.docs == "single":
        # every chunk's update has norm tau after the clip, so |S| <= k tau
        assert np.all(f64(out["alpha"]) < 1.0)


@pytest.mark.parametrize("C", synth.STACK_CHUNK_SIZES)
def test_full_size_stack(C):
    """The 6-layer stack (residual H_{l+1} = H_l + O_l, same X0) at 4 x 16384 tokens;
    the oracle reproduces the first two chunks of row 0 through all six layers."""
    w = synth.WORKLOADS["stack6_4x16k"].replace(C=C)
    dev = torch.device("cuda")
    cfg = ip.LayerConfig(B=w.B, T=w.T, d=w.d, F=w.F, C=w.C, eta=w.eta, clip=w.clip)
    layers = [stack_inputs(w, l) for l in range(w.layers)]
    X0 = layers[0]["X0"].to(dev)
    H = layers[0]["H"].to(dev)
    ws = ip.alloc_workspace(cfg, dev)
    Ds = []
    for l in range(w.layers):
        t = {k: layers[l][k].to(dev) for k in WEIGHTS}
        out = ip.forward(cfg, H, X0, *(t[k] for k in WEIGHTS), None, workspace=ws, debug=("D",), residual=True)
        Ds.append(out["D"][0, :PREFIX_CHUNKS * C].cpu())
        H = out["O"]
    torch.cuda.synchronize()
    assert ip.get_status() == 0
    Hgpu = H.cpu()
    del ws, H, X0
    torch.cuda.empty_cache()
    assert torch.isfinite(Hgpu.float()).all()
    n = PREFIX_CHUNKS * C
    params = [{k: layers[l][k].double().numpy() for k in WEIGHTS} for l in range(w.layers)]
    Hfin, outs = orc.stack_forward(params, layers[0]["X0"][:1, :n].double().numpy(),
                                   layers[0]["H"][:1, :n].double().numpy(), C, [], w.eta, w.clip)
    assert maxrel(f64(Hgpu[0, :n]), Hfin[0]) <= TOL_O
    for l in range(w.layers):
        assert normrel(f64(Ds[l]), outs[l]["D"][0]) <= 5e-2
