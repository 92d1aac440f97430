"""Context-parallel forward without a GPU: the library's host plan (ipttt_cp_plan)
and the exchange (cp_exchange over gloo), with the shard forwards done by the fp64
oracle.  Splitting a sequence over ranks, computing each shard from a zero state,
exchanging the shard aggregates once and adding the segmented exclusive sum of
the earlier ones to the continuing document's rows must give the single-sequence
forward (lijianxiong.blog notes "In-Place Test-Time Training", 工程实现: chunk
deltas in parallel, then a prefix sum; iplexlaw.co.kr review §6: exclusive scan,
reset at documents)."""
import ctypes
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from chunk_wise_weight_gate_b200 import ipttt as ip
from oracle import ipttt_oracle as fw

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

B, TL, d, F, C = 2, 192, 128, 128, 64
ETA, TAU = 0.05, 0.0


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def cfg_for(T=TL, C_=C, B_=B):
    return ip.LayerConfig(B=B_, T=T, d=d, F=F, C=C_, eta=ETA, clip=TAU)


def brute_plan(B_, T, C_, world, rank, docs):
    """The plan restated: per row, where this shard's first start is and which
    earlier shard last held a start."""
    Tg = T * world
    k = -(-T // C_)
    local, plan = [], {"row_cont": [], "first_rank": [], "prefix_chunks": [], "keep": []}
    starts = [[] for _ in range(B_)]
    for g in docs:
        starts[g // Tg].append(g % Tg)
    for b in range(B_):
        mine = [t - rank * T for t in starts[b] if rank * T <= t < (rank + 1) * T]
        local += [b * T + t for t in mine]
        owners = [0] + [t // T for t in starts[b] if t // T < rank]
        at0 = rank == 0 or (mine and mine[0] == 0)
        plan["row_cont"].append(0 if at0 else 1)
        plan["first_rank"].append(0 if rank == 0 else max(owners))
        plan["prefix_chunks"].append(0 if at0 else (mine[0] // C_ + 1 if mine else k))
        plan["keep"].append(1 if (not at0 and not mine) else 0)
    return local, plan


def random_docs(rng, B_, Tg, n):
    return sorted(set(int(x) for x in rng.integers(1, B_ * Tg, size=n)))


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_plan_matches_brute_force(world):
    rng = np.random.default_rng(world)
    cfg = cfg_for()
    Tg = TL * world
    cases = [[], [TL * (world - 1)], [Tg + TL * r for r in range(world)]]
    cases += [random_docs(rng, B, Tg, n) for n in (1, 3, 8, 30)]
    for docs in cases:
        for rank in range(world):
            assert ip.cp_plan(cfg, world, rank, docs) == brute_plan(B, TL, C, world, rank, docs), (docs, rank)


def test_plan_rejects_bad_arguments():
    cfg = cfg_for()
    for world, rank, docs in ((0, 0, []), (2, 2, []), (2, -1, []), (2, 0, [5, 5]), (2, 0, [7, 3]),
                              (2, 0, [-1]), (2, 0, [B * TL * 2])):
        with pytest.raises(ip.IptttError):
            ip.cp_plan(cfg, world, rank, docs)
    with pytest.raises(ip.IptttError):  # shards must be whole chunks when world > 1
        ip.cp_plan(cfg_for(T=TL, C_=128), 2, 0, [])
    ip.cp_plan(cfg_for(T=TL, C_=128), 1, 0, [])  # one rank: a ragged last chunk is fine


def test_cp_calls_reject_before_touching_the_device():
    cfg = cfg_for()
    # the context-parallel workspace holds a bf16 copy of every chunk's state (k + 1 of them)
    k = (cfg.T + cfg.C - 1) // cfg.C
    assert ip.cp_workspace_size(cfg) >= (k + 1) * cfg.B * cfg.d * cfg.F * 2
    f32 = ip.LayerConfig(B=1, T=64, d=8, F=8, C=16, eta=0.1, dtype="f32")
    assert ip.lib().ipttt_cp_workspace_size(ctypes.byref(f32.params())) == 0
    # null tensors are refused synchronously with IPTTT_ERR_ARG
    p = cfg.params()
    rc = ip.lib().ipttt_cp_begin(ctypes.byref(p), 2, 0, None, 0, None, None, None, None, None, None, None, None, 0,
                                 None)
    assert rc == 1
    rc = ip.lib().ipttt_cp_finish(ctypes.byref(p), 2, 0, None, 0, None, None, None, None, None, None, 0, None)
    assert rc == 1


def draw(seed, world):
    r = np.random.default_rng(seed)
    Tg = TL * world
    return {
        "H": r.standard_normal((B, Tg, d)) * 0.5,
        "X0": r.standard_normal((B, Tg, d)),
        "Wgate": r.standard_normal((F, d)) / np.sqrt(d),
        "Wup": r.standard_normal((F, d)) / np.sqrt(d),
        "Wdown0": r.standard_normal((d, F)) / np.sqrt(F),
        "conv_w": r.standard_normal((d, 5)) * 0.3,
        "Wtarget": r.standard_normal((d, d)) / np.sqrt(d),
    }


def median_chunk_norm(inp, world, docs):
    """The median ||eta P_i|| over the chunks of the whole sequence: a threshold at
    which about half the chunks clip."""
    Tg = TL * world
    flags = fw.start_flags(B, Tg, docs)
    norms = []
    for b in range(B):
        Z = fw.gated_activation(inp["H"][b], inp["Wgate"], inp["Wup"])
        V = fw.lm_target(inp["X0"][b], inp["conv_w"], inp["Wtarget"], C, flags[b])
        for (s, e, f, l, cont, has_start) in fw.chunk_segments(flags[b], C):
            norms.append(np.linalg.norm(fw.hebbian_delta(Z[l:e], V[l:e], ETA)))
    return float(np.median(norms))


def shard_forward(inp, world, rank, docs, tau=TAU):
    """One rank: the oracle forward of the shard from a zero state, the first chunk
    continuing the row's document where the plan says so, then the exchange, then
    the incoming state on the rows before the shard's first start."""
    cfg = cfg_for()
    local, plan = ip.cp_plan(cfg, world, rank, docs)
    sl = slice(rank * TL, (rank + 1) * TL)
    O = np.zeros((B, TL, d))
    S_loc = np.zeros((B, d, F))
    Z_all = np.zeros((B, TL, F))
    for b in range(B):
        flags = np.zeros(TL, dtype=bool)
        flags[0] = plan["row_cont"][b] == 0
        for g in local:
            if g // TL == b:
                flags[g % TL] = True
        Z = fw.gated_activation(inp["H"][b, sl], inp["Wgate"], inp["Wup"])
        V = fw.lm_target(inp["X0"][b, sl], inp["conv_w"], inp["Wtarget"], C, flags)
        O[b], _, S_loc[b], _ = fw.core_sequential(Z, V, inp["Wdown0"], C, flags, ETA, tau)
        Z_all[b] = Z
    gathered = ip.cp_exchange(torch.from_numpy(S_loc)).numpy()
    assert gathered.shape == (world, B, d, F)
    np.testing.assert_array_equal(gathered[rank], S_loc)
    S_final = np.zeros((B, d, F))
    for b in range(B):
        S_in = gathered[plan["first_rank"][b]:rank, b].sum(axis=0)
        if plan["row_cont"][b]:
            first = [g % TL for g in local if g // TL == b]
            end = first[0] if first else TL
            O[b, :end] += Z_all[b, :end] @ S_in.T
        S_final[b] = S_loc[b] + (S_in if plan["keep"][b] else 0.0)
    return O, S_final


def _worker(rank, world, port, docs, tau, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = draw(7, world)
        O, S_final = shard_forward(inp, world, rank, docs, tau)
        out[rank] = (O, S_final)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,docs,clip", [
    (2, [], False),                                  # one document over both shards
    (2, [TL, 2 * TL + 50], False),                   # row 0 restarts on the shard boundary; row 1 inside shard 0
    (3, [100, 3 * TL + TL + 70], False),             # row 0: start in shard 0 carries into 1 and 2
    (3, [TL + 10, 2 * TL + 64, 3 * TL + 5], False),  # starts inside shards, one on a chunk boundary
    (3, [100, 3 * TL + TL + 70], True),              # the clip active on about half the chunks
])
def test_context_parallel_equals_single_sequence(world, docs, clip):
    inp = draw(7, world)
    tau = median_chunk_norm(inp, world, docs) if clip else TAU
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, free_port(), docs, tau, out), nprocs=world, join=True)
        res = dict(out)
    full = fw.layer_forward(inp["H"], inp["X0"], inp["Wgate"], inp["Wup"], inp["Wdown0"], inp["conv_w"],
                            inp["Wtarget"], C, docs, ETA, tau)
    if clip:
        assert np.any(full["alpha"] < 1.0) and np.any(full["alpha"] == 1.0)
    D_scale = np.max(np.abs(full["D"])) if np.any(full["D"]) else 1.0
    for r in range(world):
        O, S_final = res[r]
        ref = full["O"][:, r * TL:(r + 1) * TL]
        assert np.max(np.abs(O - ref)) <= 1e-10 * max(D_scale, 1.0)
    # the last rank's state is the state after the whole sequence
    np.testing.assert_allclose(res[world - 1][1], full["S_final"], rtol=1e-10, atol=1e-12)
    # the case is one where the carried state matters
    assert D_scale > 1e-3


def test_binding_refuses_host_tensors_and_wrong_shapes():
    # the product path has no CPU fallback: host tensors are refused before any call
    cfg = cfg_for()
    H = torch.zeros(B, TL, d, dtype=torch.bfloat16)
    Wg = torch.zeros(F, d, dtype=torch.bfloat16)
    cw = torch.zeros(d, 5, dtype=torch.bfloat16)
    Wt = torch.zeros(d, d, dtype=torch.bfloat16)
    agg = torch.zeros(B, d, F)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):
        ip.cp_begin(cfg, 2, 0, H, H, Wg, Wg, cw, Wt, [], agg=agg, workspace=ws)
    with pytest.raises(ValueError, match="gathered"):
        ip.cp_finish(cfg, 2, 0, H, Wg.T.contiguous(), torch.zeros(3, B, d, F), ws, [])
    with pytest.raises(ValueError, match="shape"):
        ip.cp_begin(cfg, 2, 0, H[:, :64], H, Wg, Wg, cw, Wt, [], agg=agg, workspace=ws)
