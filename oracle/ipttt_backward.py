"""fp64 CPU oracle for the gradients of the In-Place TTT MLP layer (the backward pass).

TEST INFRASTRUCTURE ONLY, like the forward oracle (ipttt_oracle.py), whose forward
definitions it uses.  The pages give the forward but no backward formulas, though the
model is trained with the layer in place (continual training of the inserted conv
and projection from a near-zero start: cloud.tencent.com "榨干MLP的剩余价值",
验证模块一, 初始化技巧 and 两阶段增量训练流; admirer.cn article, 七、技術實現的精妙細節).  The gradients
below are derived here by the chain rule through the forward of
lijianxiong.blog notes "In-Place Test-Time Training", 方法 (gated MLP, apply, update,
LM-aligned target), the clip of cloud.tencent.com "榨干MLP的剩余价值", 详细步骤 4, and
the exclusive scan with document resets of the iplexlaw.co.kr review, §3 and §6.
Every gradient is pinned by central finite differences of the forward oracle
(tests/test_oracle_backward.py).

Per row, with A = H Wgate^T, Bu = H Wup^T, Z = SiLU(A) * Bu, U = masked conv(X0),
V = U Wtarget and, per chunk i with first segment [s, f), last segment [l, e):
    O[s:e] = Z[s:e] W0^T,  O[s:f] += Z[s:f] S_i^T when the chunk continues a document,
    P_i = V[l:e]^T Z[l:e],  dW_i = a_i eta P_i,  a_i = clip(||eta P_i||),
    S_{i+1} = keep_i S_i + dW_i.
Given upstream gradients gO = dL/dO (and optionally gS = dL/dS_final):
    gW0 = gO^T Z;  gZ = gO W0 (+ gO[s:f] S_i on continued rows);
    reverse over chunks, g = dL/dS_{i+1}:
        gP_i = eta g                                   (delta not clipped)
             = tau (g - Phat <Phat, g>) / ||P_i||      (clipped: dW_i = tau P_i / ||P_i||)
        gV[l:e] += Z[l:e] gP_i^T,  gZ[l:e] += V[l:e] gP_i,
        dL/dS_i = (keep_i ? g : 0) + gO[s:f]^T Z[s:f] (continued rows);
    gA = gZ * Bu * SiLU'(A),  gBu = gZ * SiLU(A),  SiLU'(x) = s(x)(1 + x(1 - s(x)));
    gH = gA Wgate + gBu Wup,  gWgate = gA^T H,  gWup = gBu^T H;
    gU = gV Wtarget^T,  gWtarget = U^T gV;
    U[t,c] = sum_o w[c,o] X0[t+o,c] m(t,o):  gX0[t+o,c] += w[c,o] gU[t,c] m(t,o),
                                              gw[c,o] += X0[t+o,c] gU[t,c] m(t,o).
The clip is not differentiable where ||eta P_i|| = tau exactly; the derivative on
either side is the one used.
"""
from __future__ import annotations

import numpy as np

from oracle import ipttt_oracle as fw


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _clipped(norm, tau):
    return tau is not None and np.isfinite(tau) and tau > 0.0 and norm > tau


def _conv_mask(T, C, flags_row, o):
    """m(t, o) of the masked conv: tap o of token t is inside T, the chunk and the document."""
    did = fw.doc_ids(flags_row)
    t = np.arange(T)
    src = t + o
    ok = src < T
    ok[ok] &= (src[ok] // C) == (t[ok] // C)
    ok[ok] &= did[src[ok]] == did[t[ok]]
    return ok


def row_backward(H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, C, flags_row, eta, tau, gO, gS_final=None):
    """Gradients of one row: (gH, gX0, gWgate, gWup, gWdown0, gconv_w, gWtarget)."""
    T, d = H.shape
    F = Wgate.shape[0]
    A = H @ Wgate.T
    Bu = H @ Wup.T
    Z = fw.silu(A) * Bu
    U = fw.conv_target_input(X0, conv_w, C, flags_row)
    V = U @ Wtarget
    segs = fw.chunk_segments(flags_row, C)

    # forward scan, keeping the state before each chunk
    S = np.zeros((d, F))
    states, deltas = [], []
    for (s, e, f, l, cont, has_start) in segs:
        states.append(S)
        P = V[l:e].T @ Z[l:e]
        n = np.linalg.norm(eta * P)
        deltas.append((P, n))
        a = fw.clip_factor(n, tau)
        S = (np.zeros_like(S) if has_start else S) + a * eta * P

    gW0 = gO.T @ Z
    gZ = gO @ Wdown0
    gV = np.zeros((T, d))
    g = np.zeros((d, F)) if gS_final is None else np.array(gS_final, dtype=np.float64)
    for i in range(len(segs) - 1, -1, -1):
        s, e, f, l, cont, has_start = segs[i]
        P, n = deltas[i]
        if _clipped(n, tau):
            pn = np.linalg.norm(P)
            Phat = P / pn
            gP = tau * (g - Phat * np.sum(Phat * g)) / pn
        else:
            gP = eta * g
        gV[l:e] += Z[l:e] @ gP.T
        gZ[l:e] += V[l:e] @ gP
        g_prev = np.zeros_like(g) if has_start else g
        if cont:
            gZ[s:f] += gO[s:f] @ states[i]
            g_prev = g_prev + gO[s:f].T @ Z[s:f]
        g = g_prev

    sg = _sigmoid(A)
    gA = gZ * Bu * (sg * (1.0 + A * (1.0 - sg)))
    gBu = gZ * fw.silu(A)
    gH = gA @ Wgate + gBu @ Wup
    gWgate = gA.T @ H
    gWup = gBu.T @ H
    gU = gV @ Wtarget.T
    gWtarget = U.T @ gV
    gX0 = np.zeros_like(X0)
    gconv = np.zeros_like(conv_w)
    for o in range(fw.CONV_TAPS):
        ok = _conv_mask(T, C, flags_row, o)
        t = np.nonzero(ok)[0]
        gX0[t + o] += conv_w[:, o][None, :] * gU[t]
        gconv[:, o] += np.sum(X0[t + o] * gU[t], axis=0)
    return gH, gX0, gWgate, gWup, gW0, gconv, gWtarget


def layer_backward(H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, C, doc_starts, eta, tau, gO, gS_final=None):
    """Gradients of a batch [B, T, d] given gO = dL/dO [B, T, d] and optionally
    gS_final = dL/dS_final [B, d, F].  Returns a dict keyed like the inputs."""
    H, X0, gO = (np.asarray(a, np.float64) for a in (H, X0, gO))
    B, T, d = H.shape
    flags = fw.start_flags(B, T, doc_starts)
    out = {"H": np.zeros_like(H), "X0": np.zeros_like(X0), "Wgate": np.zeros_like(Wgate),
           "Wup": np.zeros_like(Wup), "Wdown0": np.zeros_like(Wdown0), "conv_w": np.zeros_like(conv_w),
           "Wtarget": np.zeros_like(Wtarget)}
    for b in range(B):
        gs = None if gS_final is None else gS_final[b]
        gH, gX0, gWg, gWu, gW0, gcw, gWt = row_backward(H[b], X0[b], Wgate, Wup, Wdown0, conv_w, Wtarget, C,
                                                       flags[b], eta, tau, gO[b], gs)
        out["H"][b] = gH
        out["X0"][b] = gX0
        out["Wgate"] += gWg
        out["Wup"] += gWu
        out["Wdown0"] += gW0
        out["conv_w"] += gcw
        out["Wtarget"] += gWt
    return out
