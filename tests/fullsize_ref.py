"""fp64 oracle references at the layer's full sizes, for the full-size GPU tests.

The whole-row oracle (layer_forward) would hold Z of a 128k-token row in fp64
(10 GB), so the state walk is composed here from the oracle's own functions, one
chunk at a time, in the order the oracle's sequential core takes its steps: gated
activation, masked conv target, the last segment's Hebbian delta, its clip factor,
and the state reset at a chunk holding a document start [lijianxiong.blog notes
"In-Place Test-Time Training", 步骤一/步骤二; iplexlaw.co.kr review §3, §6].
Results are cached for the test session (the single-device and context-parallel
full-size tests share them).
"""
from __future__ import annotations

import functools

import numpy as np

from chunk_wise_weight_gate_b200 import synth
from oracle import ipttt_oracle as orc

WEIGHTS = ("Wgate", "Wup", "Wdown0", "conv_w", "Wtarget")


@functools.lru_cache(maxsize=2)
def inputs(name: str):
    return synth.make_inputs(synth.WORKLOADS[name], seed=0)


@functools.lru_cache(maxsize=2)
def weights64(name: str):
    inp = inputs(name)
    return {k: inp[k].double().numpy() for k in WEIGHTS}


@functools.lru_cache(maxsize=8)
def scan_row(name: str, b: int, keep: tuple = ()):
    """Walks every chunk of row b of workload `name`.

    Returns (S_final [d,F], alpha [k], states) where states maps each chunk index
    in `keep` to (S_i, D_i): the state the chunk is applied with and the oracle's
    fast-weight term D_i [C,d] of the chunk (zero rows outside its first segment,
    or all zero when a document starts on the chunk's first token)."""
    w = synth.WORKLOADS[name]
    inp = inputs(name)
    wt = weights64(name)
    flags = orc.start_flags(w.B, w.T, inp["doc_starts"].numpy())[b]
    tau = w.clip if w.clip > 0 else np.inf
    S = np.zeros((w.d, w.F))
    alphas, states = [], {}
    for i, (s, e, f, l, cont, has_start) in enumerate(orc.chunk_segments(flags, w.C)):
        H = inp["H"][b, s:e].double().numpy()
        X0 = inp["X0"][b, s:e].double().numpy()
        Z = orc.gated_activation(H, wt["Wgate"], wt["Wup"])
        if i in keep:
            D = np.zeros((e - s, w.d))
            if cont:
                D[:f - s] = Z[:f - s] @ S.T
            states[i] = (S.copy(), D)
        V = orc.lm_target(X0, wt["conv_w"], wt["Wtarget"], w.C, flags[s:e])
        dW = orc.hebbian_delta(Z[l - s:], V[l - s:], w.eta)
        a = orc.clip_factor(np.linalg.norm(dW), tau)
        alphas.append(a)
        S = (np.zeros_like(S) if has_start else S) + a * dW
    return S, np.asarray(alphas), states
