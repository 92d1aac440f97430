"""Token-by-token decoding against the whole-sequence forward and the fp64 oracle.

A token of chunk i is output with the state committed before the chunk, and the
chunk's delta is committed when the chunk is complete, so decoding a sequence token
by token must reproduce the forward over the whole sequence: the committed states
bit for bit (both commit through the streaming path), the outputs up to the fp32
summation order of the per-token kernels (bf16 rounding of O: tolerance 1e-2 against
the forward, 2e-2 against the oracle as for every bf16 output)."""
import numpy as np
import pytest
import torch

from chunk_wise_weight_gate_b200 import ipttt as ip
from tests.gpu_util import WEIGHTS, case, maxrel, oracle, to_np

pytestmark = pytest.mark.gpu


def decode_all(cfg, inp, T, w):
    dev = torch.device("cuda")
    st = ip.DecodeState(cfg, dev)
    H = inp["H"].to(dev)
    X0 = inp["X0"].to(dev)
    docs = set(int(g) for g in inp["doc_starts"].numpy())
    out = torch.empty(cfg.B, T, cfg.d, dtype=torch.bfloat16, device=dev)
    o = torch.empty(cfg.B, cfg.d, dtype=torch.bfloat16, device=dev)
    for t in range(T):
        starts = [int(b * T + t in docs) for b in range(cfg.B)]
        st.step(H[:, t].contiguous(), X0[:, t].contiguous(), *(w[k] for k in WEIGHTS), starts if any(starts) else None,
                o=o)
        out[:, t] = o
    torch.cuda.synchronize()
    assert ip.get_status() == 0
    return st, out


def test_decode_equals_forward_and_oracle():
    # no clip and a large eta make the fast-weight term 10-25% of O; documents start
    # inside chunks, on a chunk boundary and in the second row; the last chunk is short
    B, T, C = 2, 777, 128
    cfg, inp = case(B, T, C, 256, 512, eta=2e-2, clip=0.0, docs=[100, 256, 300, T + 5, T + 640])
    dev = torch.device("cuda")
    w = {k: inp[k].to(dev) for k in WEIGHTS}
    _, out = decode_all(cfg, inp, T, w)
    ref = ip.forward(cfg, inp["H"].to(dev), inp["X0"].to(dev), *(w[k] for k in WEIGHTS), inp["doc_starts"])
    torch.cuda.synchronize()
    assert maxrel(to_np(out), to_np(ref)) <= 1e-2
    orc = oracle(cfg, inp)
    assert maxrel(to_np(out), orc["O"]) <= 2e-2
    # the fast-weight term is visible: without it decode would miss the oracle
    assert maxrel(orc["O"] - orc["D"], orc["O"]) > 5 * 2e-2


@pytest.mark.parametrize("B", [1, 3])
def test_decode_one_and_three_rows(B):
    # the CUDA-core kernels below four rows, at their smallest and largest batch;
    # a document starts inside the first chunk of the last row
    T, C = 300, 128
    cfg, inp = case(B, T, C, 256, 512, eta=2e-2, clip=0.0, docs=[(B - 1) * T + 90])
    dev = torch.device("cuda")
    w = {k: inp[k].to(dev) for k in WEIGHTS}
    _, out = decode_all(cfg, inp, T, w)
    ref = ip.forward(cfg, inp["H"].to(dev), inp["X0"].to(dev), *(w[k] for k in WEIGHTS), inp["doc_starts"])
    torch.cuda.synchronize()
    assert maxrel(to_np(out), to_np(ref)) <= 1e-2
    orc = oracle(cfg, inp)
    assert maxrel(to_np(out), orc["O"]) <= 2e-2
    assert maxrel(orc["O"] - orc["D"], orc["O"]) > 5 * 2e-2


def test_decode_batched_rows_on_the_tensor_cores():
    # 8 rows: the gate/up products run as tcgen05 GEMMs (rows padded to 32); the
    # outputs match the forward and the oracle as for 2 rows
    B, T, C = 8, 300, 128
    docs = [b * T + 37 * b for b in range(1, B)] + [60, T + 200]
    cfg, inp = case(B, T, C, 256, 512, eta=2e-2, clip=0.0, docs=sorted(set(docs)))
    dev = torch.device("cuda")
    w = {k: inp[k].to(dev) for k in WEIGHTS}
    _, out = decode_all(cfg, inp, T, w)
    ref = ip.forward(cfg, inp["H"].to(dev), inp["X0"].to(dev), *(w[k] for k in WEIGHTS), inp["doc_starts"])
    torch.cuda.synchronize()
    assert maxrel(to_np(out), to_np(ref)) <= 1e-2
    orc = oracle(cfg, inp)
    assert maxrel(to_np(out), orc["O"]) <= 2e-2
    assert maxrel(orc["O"] - orc["D"], orc["O"]) > 5 * 2e-2


def test_decode_commits_the_prefill_state():
    # chunks of 512 tokens: a one-call forward then also scans chunk by chunk, as
    # the decode commits do (shorter chunks are scanned in groups of 512 tokens,
    # which agree with chunk-by-chunk commits up to rounding)
    B, C = 2, 512
    T = 3 * C
    cfg, inp = case(B, T, C, 256, 512, eta=1e-3, clip=1e-5, docs=[300, T + 20])
    dev = torch.device("cuda")
    w = {k: inp[k].to(dev) for k in WEIGHTS}
    st, _ = decode_all(cfg, inp, T, w)
    full = ip.forward(cfg, inp["H"].to(dev), inp["X0"].to(dev), *(w[k] for k in WEIGHTS), inp["doc_starts"],
                      debug=("S_final",))
    torch.cuda.synchronize()
    assert torch.equal(st.export(), full["S_final"])


def test_decode_rejects_unsupported_batches():
    with pytest.raises(ValueError):
        ip.DecodeState(ip.LayerConfig(B=17, T=1, d=256, F=512, C=128, eta=1e-3, clip=0.0))
