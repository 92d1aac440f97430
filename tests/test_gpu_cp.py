"""Context-parallel forward (ipttt_cp_begin / ipttt_cp_finish) on one GPU.

The ranks run one after another in this process, each with its own workspace;
the aggregates stacked in rank order stand in for the all-gather (the exchange
itself, cp_exchange, is covered over gloo in test_cp_host.py).  No kernel waits
on another rank, so this is the same device work each rank does.

Bars: with one rank, or on rank 0, the result is the single-device forward's, bit
for bit (same kernels, same rounding).  On later ranks the incoming state is added
to each continuing chunk's bf16 state copy (one more rounding), so O matches the
single-device forward to 1e-2 max-relative, and (where that part is large) the
difference stays within 2e-2 of the fast-weight part's norm; against the oracle the bf16 bar of 2e-2 holds.  S_final is
an fp32 sum in another order: 1e-5 normwise against the single-device state.
"""
import numpy as np
import pytest
import torch

from chunk_wise_weight_gate_b200 import ipttt as ip
from tests.gpu_util import WEIGHTS, case, maxrel, normrel, oracle, to_np

pytestmark = pytest.mark.gpu

TOL_O = 2e-2


def shard_cfg(cfg, world):
    return ip.LayerConfig(B=cfg.B, T=cfg.T // world, d=cfg.d, F=cfg.F, C=cfg.C, eta=cfg.eta, clip=cfg.clip)


def cp_emulated(cfg, inp, world, residual=False):
    """Every rank's begin, the aggregates in rank order, every rank's finish."""
    dev = torch.device("cuda")
    sc = shard_cfg(cfg, world)
    TL = sc.T
    w = {k: inp[k].to(dev) for k in WEIGHTS}
    docs = inp["doc_starts"].tolist()
    H, X0 = inp["H"].to(dev), inp["X0"].to(dev)
    ranks = []
    for r in range(world):
        Hr = H[:, r * TL:(r + 1) * TL].contiguous()
        X0r = X0[:, r * TL:(r + 1) * TL].contiguous()
        agg, ws = ip.cp_begin(sc, world, r, Hr, X0r, w["Wgate"], w["Wup"], w["conv_w"], w["Wtarget"], docs)
        ranks.append((Hr, agg, ws))
    gathered = torch.stack([agg for _, agg, _ in ranks])
    outs, finals = [], []
    for r, (Hr, _, ws) in enumerate(ranks):
        O, Sf = ip.cp_finish(sc, world, r, Hr, w["Wdown0"], gathered, ws, docs, S_final=True, residual=residual)
        outs.append(O)
        finals.append(Sf)
    torch.cuda.synchronize()
    assert ip.get_status() == 0
    return torch.cat(outs, dim=1), finals


def single(cfg, inp, residual=False):
    dev = torch.device("cuda")
    t = {k: inp[k].to(dev) for k in ("H", "X0") + WEIGHTS}
    out = ip.forward(cfg, *(t[k] for k in ("H", "X0") + WEIGHTS), inp["doc_starts"], debug=("D", "S_final"),
                     residual=residual)
    torch.cuda.synchronize()
    assert ip.get_status() == 0
    return out


def prefix_state(cfg, inp, T_end):
    """S_final of the single-device forward over the first T_end tokens of every row."""
    Tg = cfg.T
    docs = [b * T_end + t for g in inp["doc_starts"].tolist() for b, t in [divmod(g, Tg)] if t < T_end]
    sub = {k: inp[k] for k in WEIGHTS}
    sub["H"] = inp["H"][:, :T_end].contiguous()
    sub["X0"] = inp["X0"][:, :T_end].contiguous()
    sub["doc_starts"] = torch.as_tensor(np.asarray(docs, dtype=np.int32))
    pc = ip.LayerConfig(B=cfg.B, T=T_end, d=cfg.d, F=cfg.F, C=cfg.C, eta=cfg.eta, clip=cfg.clip)
    return single(pc, sub)["S_final"]


CASES = {
    # a document over all shards, the carried state large (no clip)
    "one_doc_world4": dict(world=4, B=1, T=2048, C=128, d=256, F=512, eta=2e-2, clip=0.0, docs=[]),
    # row 0: starts inside shard 1 and on the shard 1/2 boundary; row 1: shards 1, 2
    # continue shard 0's document, shard 3 starts one inside its last chunk
    "docs_world4": dict(world=4, B=2, T=2048, C=128, d=256, F=512, eta=2e-2, clip=0.0,
                        docs=[600, 1024, 2048 + 1500, 2048 + 1900]),
    # 256-token chunks (the CTA-pair Gram pass), three ranks, a start on a chunk boundary
    "chunk256_world3": dict(world=3, B=2, T=1536, C=256, d=256, F=512, eta=2e-2, clip=0.0,
                            docs=[700, 1536 + 512]),
    # the clip active, 1024-token chunks
    "clip_chunk1024_world2": dict(world=2, B=1, T=4096, C=1024, d=256, F=512, eta=1e-3, clip=1e-5, docs=[]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_cp_matches_single_device_and_oracle(name):
    kw = dict(CASES[name])
    world = kw.pop("world")
    cfg, inp = case(**kw)
    O, finals = cp_emulated(cfg, inp, world)
    ref = single(cfg, inp)
    O_np, O_ref, D_ref = to_np(O), to_np(ref["O"]), to_np(ref["D"])
    assert maxrel(O_np, O_ref) <= 1e-2
    if cfg.clip == 0:
        # where the fast-weight part is large, the difference is small against it
        # (normwise: a one-ulp flip of a large O element is several % of max |D|;
        # with the clip on, D is ~1e-7 of O and a single flip outweighs it)
        assert np.linalg.norm(O_np - O_ref) <= 2e-2 * np.linalg.norm(D_ref)
    TL = cfg.T // world
    # rank 0 sees no incoming state: the single-device result bit for bit
    assert torch.equal(O[:, :TL].cpu(), ref["O"][:, :TL].cpu())
    orc = oracle(cfg, inp)
    assert maxrel(O_np, orc["O"]) <= TOL_O
    assert normrel(to_np(finals[-1]), to_np(ref["S_final"])) <= 1e-5
    assert normrel(to_np(finals[-1]), orc["S_final"]) <= TOL_O
    for r in range(world - 1):
        assert normrel(to_np(finals[r]), to_np(prefix_state(cfg, inp, (r + 1) * TL))) <= 1e-5
    if cfg.clip == 0:
        # the carried state changes O well beyond the tolerance, so O checks it
        assert maxrel(orc["O"] - orc["D"], orc["O"]) > 5 * TOL_O


@pytest.mark.parametrize("C", [128, 256])
def test_cp_one_rank_is_the_single_device_forward(C):
    cfg, inp = case(2, 1000 if C == 128 else 1024, C, 256, 512, eta=2e-2, clip=0.0, docs=[300, 1000 + 200])
    O, finals = cp_emulated(cfg, inp, 1)
    ref = single(cfg, inp)
    assert torch.equal(O.cpu(), ref["O"].cpu())
    assert torch.equal(finals[0].cpu(), ref["S_final"].cpu())


def test_cp_residual():
    cfg, inp = case(1, 1024, 128, 256, 512, eta=2e-2, clip=0.0, docs=[])
    O, _ = cp_emulated(cfg, inp, 2, residual=True)
    ref = single(cfg, inp, residual=True)
    assert maxrel(to_np(O), to_np(ref["O"])) <= 1e-2


def test_cp_shards_starting_documents_need_no_exchange():
    # every shard starts a document in every row: each shard is an independent
    # forward, so every rank's result is bit for bit the single-device one
    world, TL = 2, 512
    cfg, inp = case(2, world * TL, 128, 256, 512, eta=2e-2, clip=0.0,
                    docs=[TL, world * TL + TL])
    O, _ = cp_emulated(cfg, inp, world)
    ref = single(cfg, inp)
    assert torch.equal(O.cpu(), ref["O"].cpu())
