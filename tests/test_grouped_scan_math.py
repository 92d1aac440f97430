"""The grouped chunk scan, restated in numpy, equals the oracle's chunk-by-chunk
scan (no GPU).

For chunks of 64 or 128 tokens the library scans G consecutive chunks at a time
(a group of 256 tokens): the state is carried, snapshotted and applied per group,
and the chunks of a group see each other's deltas through a within-group term

    E[t] = sum_{u in an earlier chunk of t's group, in t's document} (z_t . z_u) v'_u,
    v'_u = alpha(chunk(u)) eta v_u on the rows of each chunk's last segment (0 elsewhere).

The apply is linear in the state and each delta is clipped on its own, so this is
the exclusive scan of lijianxiong.blog notes "In-Place Test-Time Training",
工程实现, regrouped; iplexlaw.co.kr review §6 (reset per document).  The group
is described with the same per-chunk metadata as a chunk (first-segment end,
last-segment start, continues, has-start), computed at the group's length.
"""
import numpy as np
import pytest

from oracle import ipttt_oracle as orc


def grouped_scan(Z, V, W0, C, G, flags, eta, tau):
    T, F = Z.shape
    d = W0.shape[0]
    did = orc.doc_ids(flags)
    chunk = np.arange(T) // C
    # per chunk: clip factor, and v' on the rows of the chunk's last segment
    Vp = np.zeros_like(V)
    alphas = []
    for (s, e, f, l, cont, has_start) in orc.chunk_segments(flags, C):
        a = orc.clip_factor(np.linalg.norm(orc.hebbian_delta(Z[l:e], V[l:e], eta)), tau)
        alphas.append(a)
        Vp[l:e] = a * eta * V[l:e]
    O = Z @ W0.T
    D = np.zeros((T, d))
    S = np.zeros((d, F))
    for (s, e, f, l, cont, has_start) in orc.chunk_segments(flags, C * G):
        if cont:                                   # the group's first segment sees the carried state
            D[s:f] += Z[s:f] @ S.T
        for t in range(s, e):                      # within-group term
            u = np.arange(s, e)
            m = (chunk[u] < chunk[t]) & (did[u] == did[t])
            D[t] += ((Z[u[m]] @ Z[t])[:, None] * Vp[u[m]]).sum(axis=0)
        # the group's update: v' rows from the group's last document start on
        S = (np.zeros_like(S) if has_start else S) + Vp[l:e].T @ Z[l:e]
    return O + D, D, S, np.asarray(alphas)


@pytest.mark.parametrize("seed", range(24))
def test_grouped_scan_equals_the_chunk_scan(seed):
    rng = np.random.default_rng(seed)
    T = int(rng.integers(5, 70))
    C = int(rng.integers(1, 6))
    G = int(rng.integers(1, 5))
    d, F = 3, 5
    Z = rng.standard_normal((T, F))
    V = rng.standard_normal((T, d))
    W0 = rng.standard_normal((d, F))
    starts = sorted(set(int(x) for x in rng.integers(1, T, int(rng.integers(0, 5)))))
    flags = orc.start_flags(1, T, starts)[0]
    tau = (0.0, 0.4)[seed % 2]
    ref = orc.core_sequential(Z, V, W0, C, flags, 0.3, tau)
    got = grouped_scan(Z, V, W0, C, G, flags, 0.3, tau)
    for a, b, name in zip(got, ref, ("O", "D", "S_final", "alpha")):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12, err_msg=name)


def test_group_of_one_chunk_is_the_chunk_scan_and_the_term_vanishes():
    rng = np.random.default_rng(7)
    T, C = 40, 4
    Z, V, W0 = rng.standard_normal((T, 6)), rng.standard_normal((T, 3)), rng.standard_normal((3, 6))
    flags = orc.start_flags(1, T, [9, 22])[0]
    ref = orc.core_sequential(Z, V, W0, C, flags, 0.2, 0.0)
    got = grouped_scan(Z, V, W0, C, 1, flags, 0.2, 0.0)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
