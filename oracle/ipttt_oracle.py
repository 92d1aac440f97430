"""fp64 CPU oracle for the In-Place TTT chunk-wise fast-weight gated-MLP forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with the
CUDA path: it is the plain definition of the layer, written out in numpy float64
(library matmuls serve as steps; nothing is blocked, fused or reordered).

Sources (page title, then section / equation):
  [N]  lijianxiong.blog notes "In-Place Test-Time Training", 方法:
       gated MLP O = (phi(H Wgate^T) * (H Wup^T)) Wdown^T;  Z = phi(H Wgate^T) * (H Wup^T);
       step 1 apply  O_[i] = Z_[i] (W^(i))^T;  step 2 update W^(i+1) = W^(i) - eta grad L;
       LM-aligned target V = Conv1D(X0) Wtarget;  loss L = -<.,.>_F;
       Hebbian rule  W <- W + eta V_[i]^T Z_[i];  工程实现: cumulative form and the
       prefix sum  dS_i = sum_{j<i} dW_j (exclusive).
  [T]  cloud.tencent.com "榨干MLP的剩余价值", 详细步骤 3 (depthwise conv, kernel 5,
       no look past the chunk) and 4 (Frobenius clip of the update at 1e-5).
  [R]  iplexlaw.co.kr review of 2604.06169, §3 (apply before update: a chunk's output
       always uses the pre-update weight), §6 (exclusive scan, chunk-boundary masking,
       reset of the fast weight at each document, clip 1e-5, depthwise Conv1D size 5).

Readings taken where the pages are silent or disagree (each also listed in the
design notes):
  * Exclusive scan: chunk i is applied with W0 + sum of the deltas of chunks j < i.
  * The conv taps look at the current and the next four tokens: tap o multiplies
    X0[t+o]; a tap is zero when t+o lies past the chunk end, past T, or in another
    document.  No bias.
  * V = U @ Wtarget (literal orientation).
  * dW = +eta V^T Z  (gradient of L(W) = -<Z W^T, V>_F is -V^T Z).
  * Clip: per chunk (per segment), after eta; when ||dW||_F > tau the delta is
    scaled to norm tau.  tau <= 0 or inf: no clip.
  * Documents: a row start is a document start.  The chunk grid is fixed per row.
    Tokens of a document that started inside chunk i use W0 only; only the chunk's
    last segment (the document that runs on into chunk i+1) feeds the state, and a
    chunk containing any document start resets the state before adding that delta.
  * phi = SiLU.

All functions take and return float64 numpy arrays.
"""
from __future__ import annotations

import numpy as np

CONV_TAPS = 5


def silu(x):
    """phi of the gated MLP: x * sigmoid(x), in float64."""
    return x / (1.0 + np.exp(-x))


def start_flags(B, T, doc_starts):
    """Bool [B, T]: True where a document starts.  Row starts are always starts."""
    f = np.zeros((B, T), dtype=bool)
    f[:, 0] = True
    for g in np.asarray(doc_starts, dtype=np.int64).ravel():
        f[g // T, g % T] = True
    return f


def doc_ids(flags_row):
    """Document index of every token of one row."""
    return np.cumsum(flags_row.astype(np.int64)) - 1


def gated_activation(H, Wgate, Wup):
    """Z = phi(H Wgate^T) * (H Wup^T)  [N: 原地自适应]."""
    return silu(H @ Wgate.T) * (H @ Wup.T)


def conv_target_input(X0, conv_w, C, flags_row):
    """U[t, c] = sum_o conv_w[c, o] X0[t+o, c], taps masked at chunk/document ends [T: 步骤3]."""
    T, d = X0.shape
    did = doc_ids(flags_row)
    U = np.zeros((T, d))
    t = np.arange(T)
    for o in range(CONV_TAPS):
        src = t + o
        ok = src < T
        ok[ok] &= (src[ok] // C) == (t[ok] // C)
        ok[ok] &= did[src[ok]] == did[t[ok]]
        U[ok] += conv_w[:, o][None, :] * X0[src[ok]]
    return U


def lm_target(X0, conv_w, Wtarget, C, flags_row):
    """V = Conv1D(X0) Wtarget  [N: 对齐语言模型的目标函数]."""
    return conv_target_input(X0, conv_w, C, flags_row) @ Wtarget


def hebbian_delta(Z, V, eta):
    """-eta * grad_W L(Z W^T, V) with L = -<., .>_F, i.e. eta V^T Z  [N: update rule]."""
    return eta * (V.T @ Z)


def clip_factor(norm, tau):
    """Scale that brings a delta of Frobenius norm `norm` down to tau  [T: 步骤4]."""
    if tau is None or not np.isfinite(tau) or tau <= 0.0:
        return 1.0
    return tau / norm if norm > tau else 1.0


def chunk_segments(flags_row, C):
    """Per chunk: (start, end, first_seg_end, last_seg_start, continues, has_start)."""
    T = len(flags_row)
    out = []
    for s in range(0, T, C):
        e = min(s + C, T)
        starts = [t for t in range(s, e) if flags_row[t]]
        cont = not flags_row[s]
        inner = [t for t in starts if t > s]
        first_end = inner[0] if inner else e
        last_start = starts[-1] if starts else s
        out.append((s, e, first_end, last_start, cont, len(starts) > 0))
    return out


def core_sequential(Z, V, W0, C, flags_row, eta, tau):
    """Apply-then-update loop over chunks of one row  [N: 步骤一/步骤二; R: §3].

    Returns O [T,d], D [T,d] (the Z S_i^T part of O), S_final [d,F], alpha [k].
    """
    T, F = Z.shape
    d = W0.shape[0]
    O = np.zeros((T, d))
    D = np.zeros((T, d))
    S = np.zeros((d, F))
    alphas = []
    for (s, e, f, l, cont, has_start) in chunk_segments(flags_row, C):
        O[s:e] = Z[s:e] @ W0.T                     # apply with W0 ...
        if cont:                                   # ... plus the carried state for the
            D[s:f] = Z[s:f] @ S.T                  # document that runs on from chunk i-1
            O[s:f] += D[s:f]
        dW = hebbian_delta(Z[l:e], V[l:e], eta)    # update from the last segment only
        a = clip_factor(np.linalg.norm(dW), tau)
        alphas.append(a)
        S = (np.zeros_like(S) if has_start else S) + a * dW
    return O, D, S, np.asarray(alphas)


def core_prefix_sum(Z, V, W0, C, flags_row, eta, tau):
    """Parallel form: every chunk delta first, then an exclusive per-document prefix sum
    [N: 工程实现, dS_i = sum_{j<i} dW_j; R: §6 exclusive scan, document reset]."""
    T, F = Z.shape
    d = W0.shape[0]
    did = doc_ids(flags_row)
    segs = chunk_segments(flags_row, C)
    deltas, alphas, last_doc = [], [], []
    for (s, e, f, l, cont, has_start) in segs:
        dW = hebbian_delta(Z[l:e], V[l:e], eta)
        a = clip_factor(np.linalg.norm(dW), tau)
        deltas.append(a * dW)
        alphas.append(a)
        last_doc.append(did[e - 1])
    O = Z @ W0.T
    D = np.zeros((T, d))
    S_final = None
    for i, (s, e, f, l, cont, has_start) in enumerate(segs):
        if cont:
            Si = np.zeros((d, F))
            for j in range(i):
                if last_doc[j] == did[s]:
                    Si += deltas[j]
            D[s:f] = Z[s:f] @ Si.T
    # state after the last chunk: the deltas of the final document
    S_final = np.zeros((d, F))
    for j in range(len(segs)):
        if last_doc[j] == did[T - 1]:
            S_final += deltas[j]
    return O + D, D, S_final, np.asarray(alphas)


def core_bruteforce(Z, V, W0, C, flags_row, eta, tau):
    """Per-token form O[t] = z_t W0^T + sum_{s in P(t)} alpha(s) eta (z_s . z_t) v_s
    [N: 理论分析, logit expansion with learning-rate lambda], where P(t) holds the
    tokens of t's document in earlier chunks.  The clip norm comes from Gram
    matrices: ||V^T Z||_F^2 = sum_{s,s'} (v_s . v_s')(z_s . z_s')."""
    T, F = Z.shape
    d = W0.shape[0]
    did = doc_ids(flags_row)
    chunk = np.arange(T) // C
    k = int(chunk[-1]) + 1
    # alpha per chunk from the Gram form, over tokens of the chunk's last document
    alphas = np.ones(k)
    for i in range(k):
        rows = np.nonzero(chunk == i)[0]
        rows = rows[did[rows] == did[rows[-1]]]
        gv = V[rows] @ V[rows].T
        gz = Z[rows] @ Z[rows].T
        n = eta * np.sqrt(max(float(np.sum(gv * gz)), 0.0))
        alphas[i] = clip_factor(n, tau)
    O = np.zeros((T, d))
    D = np.zeros((T, d))
    for t in range(T):
        acc = np.zeros(d)
        for s in range(chunk[t] * C):
            if did[s] == did[t]:
                acc += alphas[chunk[s]] * eta * float(Z[s] @ Z[t]) * V[s]
        D[t] = acc
        O[t] = Z[t] @ W0.T + acc
    S_final = np.zeros((d, F))
    for s in range(T):
        if did[s] == did[T - 1]:
            S_final += alphas[chunk[s]] * eta * np.outer(V[s], Z[s])
    return O, D, S_final, alphas


CORES = {"sequential": core_sequential, "prefix_sum": core_prefix_sum,
         "bruteforce": core_bruteforce}


def layer_forward(H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, C, doc_starts, eta, tau,
                  form="sequential"):
    """One In-Place TTT MLP layer over a batch [B, T, d].

    Returns dict with O, D [B,T,d]; S_final [B,d,F]; alpha [B,k]; Z [B,T,F]; V [B,T,d].
    """
    H, X0 = np.asarray(H, np.float64), np.asarray(X0, np.float64)
    B, T, d = H.shape
    flags = start_flags(B, T, doc_starts)
    outs = {"O": [], "D": [], "S_final": [], "alpha": [], "Z": [], "V": []}
    for b in range(B):
        Z = gated_activation(H[b], Wgate, Wup)
        V = lm_target(X0[b], conv_w, Wtarget, C, flags[b])
        O, D, S, a = CORES[form](Z, V, Wdown0, C, flags[b], eta, tau)
        for key, val in (("O", O), ("D", D), ("S_final", S), ("alpha", a), ("Z", Z), ("V", V)):
            outs[key].append(val)
    return {k: np.stack(v) for k, v in outs.items()}


def core_forward(Z, V, Wdown0, C, doc_starts, eta, tau, form="sequential"):
    """The chunk scan alone, with Z [B,T,F] and V [B,T,d] supplied directly."""
    Z, V = np.asarray(Z, np.float64), np.asarray(V, np.float64)
    B, T, _ = Z.shape
    flags = start_flags(B, T, doc_starts)
    res = [CORES[form](Z[b], V[b], Wdown0, C, flags[b], eta, tau) for b in range(B)]
    return {"O": np.stack([r[0] for r in res]), "D": np.stack([r[1] for r in res]),
            "S_final": np.stack([r[2] for r in res]), "alpha": np.stack([r[3] for r in res])}


def stack_forward(layers, X0, H0, C, doc_starts, eta, tau):
    """Layers chained with the residual H_{l+1} = H_l + O_l, all fed the same X0."""
    H = np.asarray(H0, np.float64)
    outs = []
    for p in layers:
        r = layer_forward(H, X0, p["Wgate"], p["Wup"], p["Wdown0"], p["conv_w"], p["Wtarget"],
                          C, doc_starts, eta, tau)
        outs.append(r)
        H = H + r["O"]
    return H, outs
