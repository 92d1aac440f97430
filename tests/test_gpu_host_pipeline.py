"""ipttt_forward_host: the host-buffer forward pipelined through the streaming path
must give exactly ipttt_forward's result (streaming is exact: the conv look-ahead
and the state update stop at chunk ends and the fp32 state is carried)."""
import numpy as np
import pytest
import torch

from chunk_wise_weight_gate_b200 import ipttt as ip
from tests.gpu_util import WEIGHTS, case

pytestmark = pytest.mark.gpu


def device_forward(cfg, inp):
    dev = torch.device("cuda")
    t = {k: inp[k].to(dev) for k in ("H", "X0") + WEIGHTS}
    O = ip.forward(cfg, *(t[k] for k in ("H", "X0") + WEIGHTS), inp["doc_starts"])
    torch.cuda.synchronize()
    return O.cpu()


def host_forward(cfg, inp, piece, pinned=True):
    dev = torch.device("cuda")
    w = {k: inp[k].to(dev) for k in WEIGHTS}
    H = inp["H"].contiguous()
    X0 = inp["X0"].contiguous()
    if pinned:
        H, X0 = H.pin_memory(), X0.pin_memory()
    O = ip.forward_host(cfg, H, X0, *(w[k] for k in WEIGHTS), inp["doc_starts"], piece_tokens=piece)
    torch.cuda.synchronize()
    assert ip.get_status() == 0
    return O


@pytest.mark.parametrize("piece", [0, 512, 1024])
def test_host_pipeline_equals_device_forward(piece):
    # ragged T (last piece and last chunk short), documents inside pieces and on
    # a piece boundary, two rows; 128-token chunks are scanned in groups of 512
    # tokens, and pieces of whole groups reproduce the one-call result exactly
    cfg, inp = case(2, 777, 128, 256, 512, eta=2e-2, clip=0.0, docs=[100, 256, 300, 777 + 5, 777 + 640])
    ref = device_forward(cfg, inp)
    out = host_forward(cfg, inp, piece)
    assert torch.equal(out, ref)


@pytest.mark.parametrize("piece", [128, 256, 384])
def test_host_pipeline_pieces_of_part_groups(piece):
    """Pieces of whole chunks that split a scan group: the same result up to the
    rounding of the regrouped state sums and bf16 snapshots."""
    cfg, inp = case(2, 777, 128, 256, 512, eta=2e-2, clip=0.0, docs=[100, 256, 300, 777 + 5, 777 + 640])
    ref = device_forward(cfg, inp).double()
    out = host_forward(cfg, inp, piece).cpu().double()
    assert ((out - ref).abs().max() / ref.abs().max()).item() <= 1e-2


def test_host_pipeline_pageable_memory_and_clip():
    # 256-token chunks are scanned in groups of 512 tokens: pieces of one group
    cfg, inp = case(1, 1024, 256, 256, 512, eta=1e-3, clip=1e-5)
    ref = device_forward(cfg, inp)
    assert torch.equal(host_forward(cfg, inp, 512, pinned=False), ref)


def test_host_pipeline_rejects_bad_arguments_before_launching():
    cfg, inp = case(1, 512, 128, 256, 512, docs=[300, 200])
    dev = torch.device("cuda")
    w = {k: inp[k].to(dev) for k in WEIGHTS}
    with pytest.raises(ip.IptttError):
        ip.forward_host(cfg, inp["H"], inp["X0"], *(w[k] for k in WEIGHTS), inp["doc_starts"], piece_tokens=128)
    with pytest.raises(ValueError):
        ip.forward_host(cfg, inp["H"], inp["X0"], *(w[k] for k in WEIGHTS), None, piece_tokens=100)
    torch.cuda.synchronize()
    assert ip.get_status() == 0
