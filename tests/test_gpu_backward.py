"""Backward of the layer (ipttt_backward) against the fp64 oracle's gradients
(oracle/ipttt_backward.py, pinned by finite differences of the forward oracle).

fp32 inputs run on the CUDA cores in fp32: every gradient within 1e-4 of its norm
(normwise) and 1e-3 of its largest element (max-relative).  A gradient is a chain
of at most five fp32 products with K up to a few hundred (relative rounding about
sqrt(K) 2^-24 each, 1e-6) plus the forward's own 1e-5 bar, with a 10x margin.

bf16 inputs run on the tensor cores: bf16 operands (the forward's Z and V, the
per-chunk deltas P_i, the bf16 copies of the state gradient G_{i+1}, gA, gBu, gV)
with fp32 accumulators, so each operand carries a relative rounding of up to
2^-9 = 2e-3 and a gradient a few of them: held to 2e-2 normwise (the forward's bar
on its fast-weight term) and 5e-2 max-relative.
"""
import numpy as np
import pytest
import torch

from chunk_wise_weight_gate_b200 import ipttt as ip
from oracle import ipttt_backward as obwd
from tests.gpu_util import WEIGHTS, case, maxrel, normrel, to_np

pytestmark = pytest.mark.gpu

NAMES = ("H", "X0") + WEIGHTS

CASES = {
    # documents inside a chunk and on a chunk boundary, a one-token last chunk,
    # every chunk clipped
    "docs_clip_all": dict(B=2, T=49, C=8, d=16, F=24, dtype="f32", eta=0.05, clip=1e-4,
                          docs=[10, 16, 49 + 20, 49 + 21], conv_std=0.3, wtarget="identity_noise", gS=True),
    # no clip, the carried state large
    "noclip": dict(B=1, T=64, C=16, d=32, F=48, dtype="f32", eta=0.1, clip=0.0, docs=[],
                   conv_std=0.3, wtarget="identity_noise", gS=False),
    # bf16 on the tensor cores: documents inside chunks, some chunks clipped and some not
    # (delta norms ||eta P_i|| 8.1 .. 12.5: tau = 10 clips all but one, 19% and more from the kink)
    "bf16_docs_clip": dict(B=2, T=320, C=64, d=128, F=256, dtype="bf16", eta=0.02, clip=10.0,
                           docs=[70, 200, 320 + 33], conv_std=0.3, wtarget="identity_noise", gS=True),
    # several tiles of every product (F = 512: two 256-column tiles), a ragged last chunk
    # (delta norms 10.6 .. 17.3: tau = 15 clips two of five, 7% and more from the kink)
    "bf16_tiles_ragged": dict(B=1, T=600, C=128, d=256, F=512, dtype="bf16", eta=0.01, clip=15.0,
                              docs=[70, 333], conv_std=0.3, wtarget="identity_noise", gS=True),
    # 256-token chunks (the per-chunk-row products on CTA pairs), documents, a ragged
    # last chunk (delta norms 18.9 .. 24.8: tau = 21.8 clips three of six, 2% and more from the kink)
    "bf16_chunk256": dict(B=2, T=700, C=256, d=256, F=512, dtype="bf16", eta=0.01, clip=21.8,
                          docs=[300, 700 + 100], conv_std=0.3, wtarget="identity_noise", gS=True),
    # no clip, no gS: the reverse scan starts from zero
    "bf16_noclip": dict(B=1, T=256, C=64, d=128, F=256, dtype="bf16", eta=0.05, clip=0.0, docs=[],
                        conv_std=0.3, wtarget="identity_noise", gS=False),
}


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_the_oracle(name):
    kw = dict(CASES[name])
    with_gs = kw.pop("gS")
    cfg, inp = case(**kw)
    dev = torch.device("cuda")
    rng = np.random.default_rng(5)
    gO = torch.as_tensor(rng.standard_normal((cfg.B, cfg.T, cfg.d)), dtype=cfg.torch_dtype)
    gS = torch.as_tensor(rng.standard_normal((cfg.B, cfg.d, cfg.F)), dtype=torch.float32) if with_gs else None
    t = {k: inp[k].to(dev) for k in NAMES}
    got = ip.backward(cfg, *(t[k] for k in NAMES), inp["doc_starts"], gO.to(dev),
                      gS.to(dev) if gS is not None else None)
    torch.cuda.synchronize()
    assert ip.get_status() == 0
    a = {k: to_np(inp[k]) for k in NAMES}
    ref = obwd.layer_backward(a["H"], a["X0"], a["Wgate"], a["Wup"], a["Wdown0"], a["conv_w"], a["Wtarget"], cfg.C,
                              inp["doc_starts"].numpy(), cfg.eta, cfg.clip, to_np(gO),
                              gS.double().numpy() if gS is not None else None)
    tol_norm, tol_max = (1e-4, 1e-3) if cfg.dtype == "f32" else (2e-2, 5e-2)
    errs = {k: (normrel(to_np(got[k]), ref[k]), maxrel(to_np(got[k]), ref[k])) for k in NAMES}
    print(name, {k: f"{a:.2e}/{b:.2e}" for k, (a, b) in errs.items()})
    for k in NAMES:
        assert np.all(np.isfinite(to_np(got[k]))), k
        assert errs[k][0] <= tol_norm, (k, errs[k])
        assert errs[k][1] <= tol_max, (k, errs[k])
    if cfg.clip > 0:
        # the case reaches the clipped branch's derivative: the gradients of the
        # same layer without the clip are far outside the tolerance above
        ref0 = obwd.layer_backward(a["H"], a["X0"], a["Wgate"], a["Wup"], a["Wdown0"], a["conv_w"], a["Wtarget"],
                                   cfg.C, inp["doc_starts"].numpy(), cfg.eta, 0.0, to_np(gO),
                                   gS.double().numpy() if gS is not None else None)
        assert max(normrel(ref0[k], ref[k]) for k in NAMES) > 3 * tol_norm


def test_backward_is_deterministic():
    kw = dict(CASES["docs_clip_all"])
    kw.pop("gS")
    cfg, inp = case(**kw)
    dev = torch.device("cuda")
    gO = torch.ones(cfg.B, cfg.T, cfg.d, dtype=cfg.torch_dtype, device=dev)
    t = {k: inp[k].to(dev) for k in NAMES}
    a = ip.backward(cfg, *(t[k] for k in NAMES), inp["doc_starts"], gO)
    b = ip.backward(cfg, *(t[k] for k in NAMES), inp["doc_starts"], gO)
    for k in NAMES:
        assert torch.equal(a[k], b[k]), k
