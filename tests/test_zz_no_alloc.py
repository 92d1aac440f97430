"""ipttt_forward_noalloc gives the same result as ipttt_forward.

Some callers may not allocate device memory: their memory belongs to another
allocator (a framework's caching allocator, a serving runtime with a fixed
budget), or they run on a latency-critical path where cudaMalloc's implicit
synchronisation is not acceptable.  For them the library offers a forward that
runs the same kernels on its own static scratch array instead of a caller
workspace.  This file is collected last on purpose, so that a run that stops at
its first failure has run every other test first; it also passes on its own in a
fresh process, where its first call looks up the scratch address.
"""
import ctypes

import pytest
import torch

from chunk_wise_weight_gate_b200 import ipttt as ip
from tests.gpu_util import case, maxrel, to_np

pytestmark = pytest.mark.gpu

NAMES = ("H", "X0", "Wgate", "Wup", "Wdown0", "conv_w", "Wtarget")
TOL_O_BF16 = 2e-2


def forward_noalloc(cfg, t, docs, O):
    """Calls the C entry point directly (argument marshalling only)."""
    d = None
    n = 0
    if docs is not None and docs.numel() > 0:
        d = docs.to(device=O.device, dtype=torch.int32).contiguous()
        n = d.numel()
    rc = ip.lib().ipttt_forward_noalloc(ctypes.byref(cfg.params()), *(t[k].data_ptr() for k in NAMES),
                                        d.data_ptr() if d is not None else None, n, O.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return rc


def test_noalloc_forward_matches_forward_on_two_calls_in_a_row():
    dev = torch.device("cuda")
    # Unclipped with a large eta, so the fast-weight term is a visible part of O.
    for seed, docs in ((1, [100, 300, 512 + 200]), (2, [])):
        cfg, inp = case(2, 512, 128, 256, 512, eta=2e-2, clip=0.0, docs=docs, seed=seed)
        t = {k: inp[k].to(dev) for k in NAMES}
        ref = ip.forward(cfg, *(t[k] for k in NAMES), inp["doc_starts"])
        torch.cuda.synchronize()
        O = torch.full_like(ref, float("nan"))
        assert forward_noalloc(cfg, t, inp["doc_starts"], O) == 0
        assert ip.get_status() == 0
        assert maxrel(to_np(O), to_np(ref)) <= TOL_O_BF16
        assert torch.equal(O, ref)  # the same kernels on the same inputs


def test_noalloc_forward_rejects_shapes_beyond_its_scratch():
    cfg = ip.LayerConfig(B=1, T=131072, d=2560, F=9728, C=1024, eta=1e-3, clip=1e-5)
    assert ip.workspace_size(cfg) > (32 << 20)
    dev = torch.device("cuda")
    dummy = torch.empty(16, dtype=torch.bfloat16, device=dev)  # never read: the call stops first
    t = {k: dummy for k in NAMES}
    assert forward_noalloc(cfg, t, None, dummy) == 2  # IPTTT_ERR_SHAPE
