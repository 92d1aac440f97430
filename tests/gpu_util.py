"""Helpers shared by the GPU tests: input drawing, oracle calls, error metrics."""
import numpy as np
import torch

from chunk_wise_weight_gate_b200 import ipttt as ip
from chunk_wise_weight_gate_b200 import synth
from oracle import ipttt_oracle as orc

WEIGHTS = ("Wgate", "Wup", "Wdown0", "conv_w", "Wtarget")


def maxrel(x, ref):
    """max |x - ref| / max |ref|, the relative error the layer's tolerances use."""
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(x - ref)) / den) if den > 0 else float(np.max(np.abs(x)))


def normrel(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / den) if den > 0 else float(np.linalg.norm(x))


def case(B, T, C, d, F, dtype="bf16", eta=1e-3, clip=1e-5, docs=None, seed=0, **kw):
    """Inputs (CPU tensors) and a LayerConfig for a synthetic case."""
    w = synth.Workload("case", B=B, T=T, C=C, d=d, F=F, dtype=dtype, eta=eta, clip=clip, **kw)
    inp = synth.make_inputs(w, seed=seed)
    if docs is not None:
        inp["doc_starts"] = torch.as_tensor(np.asarray(docs, dtype=np.int32))
    cfg = ip.LayerConfig(B=B, T=T, d=d, F=F, C=C, eta=eta, clip=clip, dtype=dtype)
    return cfg, inp


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle(cfg, inp, form="sequential"):
    """Oracle outputs; V is restricted, as the library exports it, to the rows of
    each chunk's last document segment (the only rows that feed the update)."""
    a = {k: to_np(inp[k]) for k in ("H", "X0") + WEIGHTS}
    r = orc.layer_forward(a["H"], a["X0"], a["Wgate"], a["Wup"], a["Wdown0"], a["conv_w"], a["Wtarget"],
                          cfg.C, inp["doc_starts"].numpy(), cfg.eta, cfg.clip, form)
    flags = orc.start_flags(cfg.B, cfg.T, inp["doc_starts"].numpy())
    for b in range(cfg.B):
        for (s, e, f, l, cont, has_start) in orc.chunk_segments(flags[b], cfg.C):
            r["V"][b, s:l] = 0.0
    return r


def gpu(cfg, inp, debug=True, **kw):
    dev = torch.device("cuda")
    t = {k: inp[k].to(dev) for k in ("H", "X0") + WEIGHTS}
    out = ip.forward(cfg, t["H"], t["X0"], t["Wgate"], t["Wup"], t["Wdown0"], t["conv_w"], t["Wtarget"],
                     inp["doc_starts"], debug=debug, **kw)
    torch.cuda.synchronize()
    assert ip.get_status() == 0
    return out


# Largest scale error allowed on a fast-weight state, as the error's component
# along the reference state (scale_bias).  Rounding the bf16 operands turns every
# delta by a small random angle, which leaves a component of the order of the
# squared normwise error (about 1e-5 here: measured |bias| <= 1.8e-5 on the
# workloads' shapes); summing the deltas in fp32 (round to nearest) adds k u at
# most.  A state update that lets the tensor cores add each small delta onto the
# large running sum loses the addends' low bits and shrinks the state instead:
# measured -7.2e-5 over 1024 chunks.
BIAS_TOL = 4e-5


def scale_bias(x, ref):
    """<x - ref, ref> / <ref, ref>: the relative error of x along ref."""
    x, ref = np.asarray(x, np.float64).ravel(), np.asarray(ref, np.float64).ravel()
    den = float(ref @ ref)
    return float((x - ref) @ ref) / den if den > 0 else 0.0
