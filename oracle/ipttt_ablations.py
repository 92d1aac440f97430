"""fp64 CPU oracle for the ablations of the In-Place TTT MLP layer.

TEST INFRASTRUCTURE ONLY, like the forward oracle (ipttt_oracle.py), whose
definitions it reuses.  Nothing here is imported by the CUDA path.

Sources (page title, then section):
  * cloud.tencent.com "榨干MLP的剩余价值", 验证模块三 (目标组件剥离) and admirer.cn
    article, 五 (the ablation paragraph): the LM-aligned target with one of its two
    parts taken out, the depthwise conv (the look-ahead) or the projection Wtarget.
    Both are weight settings of the unchanged layer:
      without the conv:       tap 0 of every channel 1, taps 1..4 zero, so U = X0
                              (tap 0 is never masked: it reads the token itself);
      without the projection: Wtarget = I, so V = Conv1D(X0).
  * iplexlaw.co.kr review, §6: norm clipping keeps the accumulated update from
    swamping long sequences.  The pages do not fix whether the clip acts on each
    chunk's delta (the forward oracle's reading) or on the accumulated fast weight;
    the second reading is the ablation here:
      S_{i+1} = c_i (keep_i S_i + eta V_L^T Z_L),  c_i = min(1, tau / ||keep_i S_i + eta V_L^T Z_L||_F)
    with the same chunk grid, document segments and exclusive apply as the forward.

Two formulations of that recurrence: the direct one (the state itself clipped
after each chunk), and a lazily scaled one, S_i = g_i St_i, in which the state
St_i is never rescaled and the norm is carried as a scalar:
  ||keep S_i + dW_i||^2 = keep (||S_i||^2 + 2 eta g_i sum_{t in L} v_t . (St_i z_t)) + ||dW_i||^2,
  St_{i+1} = keep St_i + dW_i / h_i,  h_i = keep ? g_i : 1,  g_{i+1} = c_i h_i,
so that all one needs per chunk is the squared norm of the delta (the Gram pass)
and the dot products of V with the state applied to Z (an apply product).
"""
from __future__ import annotations

import numpy as np

from oracle import ipttt_oracle as fw


def conv_without_lookahead(d):
    """conv_w [d, 5] of the target without its conv: U = X0."""
    w = np.zeros((d, fw.CONV_TAPS))
    w[:, 0] = 1.0
    return w


def target_without_projection(d):
    """Wtarget [d, d] of the target without its projection: V = Conv1D(X0)."""
    return np.eye(d)


def core_state_clip(Z, V, W0, C, flags_row, eta, tau):
    """Apply-then-update over the chunks of one row, the accumulated state clipped.

    Returns O [T,d], D [T,d], S_final [d,F] and the per-chunk scale c [k].
    """
    T, F = Z.shape
    d = W0.shape[0]
    O = np.zeros((T, d))
    D = np.zeros((T, d))
    S = np.zeros((d, F))
    scales = []
    for (s, e, f, l, cont, has_start) in fw.chunk_segments(flags_row, C):
        O[s:e] = Z[s:e] @ W0.T
        if cont:
            D[s:f] = Z[s:f] @ S.T
            O[s:f] += D[s:f]
        new = (np.zeros_like(S) if has_start else S) + fw.hebbian_delta(Z[l:e], V[l:e], eta)
        c = fw.clip_factor(np.linalg.norm(new), tau)
        scales.append(c)
        S = c * new
    return O, D, S, np.asarray(scales)


def core_state_clip_scaled(Z, V, W0, C, flags_row, eta, tau):
    """The same recurrence with S_i = g_i St_i and the squared norm of S_i carried as a
    scalar (see the module notes).  Same returns as core_state_clip."""
    T, F = Z.shape
    d = W0.shape[0]
    O = np.zeros((T, d))
    D = np.zeros((T, d))
    St = np.zeros((d, F))
    g = 1.0
    n2 = 0.0            # ||S_i||_F^2
    scales = []
    for (s, e, f, l, cont, has_start) in fw.chunk_segments(flags_row, C):
        O[s:e] = Z[s:e] @ W0.T
        if cont:
            D[s:f] = g * (Z[s:f] @ St.T)
            O[s:f] += D[s:f]
        keep = not has_start
        dW = fw.hebbian_delta(Z[l:e], V[l:e], eta)
        d2 = float(np.sum(dW * dW))
        if keep:
            cross = eta * g * float(np.sum(V[l:e] * (Z[l:e] @ St.T)))
            m2 = n2 + 2.0 * cross + d2
        else:
            m2 = d2
        c = fw.clip_factor(np.sqrt(max(m2, 0.0)), tau)
        scales.append(c)
        h = g if keep else 1.0
        St = (St if keep else np.zeros_like(St)) + dW / h
        g = c * h
        n2 = c * c * m2
    return O, D, g * St, np.asarray(scales)


FORMS = {"direct": core_state_clip, "scaled": core_state_clip_scaled}


def layer_forward_state_clip(H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, C, doc_starts, eta, tau, form="direct"):
    """One layer over a batch [B, T, d] with the accumulated state clipped.
    Returns dict with O, D [B,T,d]; S_final [B,d,F]; scale [B,k]."""
    H, X0 = np.asarray(H, np.float64), np.asarray(X0, np.float64)
    B, T, d = H.shape
    flags = fw.start_flags(B, T, doc_starts)
    outs = {"O": [], "D": [], "S_final": [], "scale": []}
    for b in range(B):
        Z = fw.gated_activation(H[b], Wgate, Wup)
        V = fw.lm_target(X0[b], conv_w, Wtarget, C, flags[b])
        O, D, S, c = FORMS[form](Z, V, Wdown0, C, flags[b], eta, tau)
        for key, val in (("O", O), ("D", D), ("S_final", S), ("scale", c)):
            outs[key].append(val)
    return {k: np.stack(v) for k, v in outs.items()}
