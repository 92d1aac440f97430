"""The objective ablations of cloud.tencent.com "榨干MLP的剩余价值", 验证模块三
(目标组件剥离) and the admirer.cn article, 五: the LM-aligned target without its
conv or without its projection.  Both are weight settings of the unchanged layer,
so they run through the same kernels and are held to the same bars as every bf16
parity case (oracle/ipttt_ablations.py gives the weights)."""
import numpy as np
import pytest
import torch

from oracle import ipttt_ablations as ab
from tests.gpu_util import case, gpu, maxrel, normrel, oracle, to_np
from tests.test_gpu_parity import check_bf16

pytestmark = pytest.mark.gpu

CASES = {
    "clip": dict(B=2, T=1000, C=256, d=256, F=512, eta=1e-3, clip=1e-5, docs=[100, 300, 1000 + 700]),
    "noclip_stress": dict(B=2, T=777, C=128, d=256, F=512, eta=2e-2, clip=0.0, docs=[129, 500, 777 + 384]),
}


def ablate(inp, conv=True, projection=True):
    d = inp["H"].shape[-1]
    if not conv:
        inp["conv_w"] = torch.from_numpy(ab.conv_without_lookahead(d)).to(inp["conv_w"].dtype)
    if not projection:
        inp["Wtarget"] = torch.from_numpy(ab.target_without_projection(d)).to(inp["Wtarget"].dtype)
    return inp


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("part", ["conv", "projection"])
def test_target_without_one_part(name, part):
    kw = dict(CASES[name])
    cfg, inp = case(**kw)
    inp = ablate(inp, conv=part != "conv", projection=part != "projection")
    out = gpu(cfg, inp)
    check_bf16(out, oracle(cfg, inp), cfg.clip)


def test_target_without_both_parts_is_the_token_itself():
    # taps (1, 0, 0, 0, 0) and Wtarget = I: the conv and the target GEMM each add
    # exact zeros to one exact product, so V is X0 bit for bit on the rows that feed
    # the update (the last document segment of each chunk) and zero elsewhere
    cfg, inp = case(**CASES["noclip_stress"])
    inp = ablate(inp, conv=False, projection=False)
    out = gpu(cfg, inp)
    ref = oracle(cfg, inp)
    V = out["V"].cpu()
    mask = torch.from_numpy(ref["V"] != 0).any(dim=-1, keepdim=True)
    assert torch.equal(V, torch.where(mask, inp["X0"], torch.zeros_like(inp["X0"])))
    check_bf16(out, ref, cfg.clip)


# The clip on the accumulated state (iplexlaw.co.kr review, §6, read the other way):
# S_{i+1} = c_i (keep_i S_i + eta V_L^T Z_L).  fp32 path; held to the fp32 bars of
# the forward (1e-5 on O and S_final) against oracle/ipttt_ablations.py.
STATE_CLIP_CASES = {
    # documents inside chunks and on a chunk boundary, a ragged last chunk; tau
    # small enough that the state is clipped after most chunks
    "docs_ragged": dict(B=2, T=100, C=12, d=24, F=40, eta=0.05, clip=0.05, docs=[13, 36, 41, 100 + 7, 100 + 70]),
    # one document, several tiles of every product; the state first grows unclipped,
    # then is clipped from the fourth chunk on
    "tiles": dict(B=1, T=256, C=32, d=64, F=256, eta=0.01, clip=6.0, docs=[]),
}


def state_clip_oracle(cfg, inp):
    a = {k: to_np(inp[k]) for k in ("H", "X0") + ("Wgate", "Wup", "Wdown0", "conv_w", "Wtarget")}
    return ab.layer_forward_state_clip(a["H"], a["X0"], a["Wgate"], a["Wup"], a["Wdown0"], a["conv_w"],
                                       a["Wtarget"], cfg.C, inp["doc_starts"].numpy(), cfg.eta, cfg.clip)


@pytest.mark.parametrize("name", list(STATE_CLIP_CASES))
def test_state_clip(name):
    kw = dict(STATE_CLIP_CASES[name])
    cfg, inp = case(dtype="f32", conv_std=0.3, wtarget="identity_noise", **kw)
    out = gpu(cfg, inp, state_clip=True)
    ref = state_clip_oracle(cfg, inp)
    assert maxrel(to_np(out["O"]), ref["O"]) <= 1e-5
    assert normrel(to_np(out["S_final"]), ref["S_final"]) <= 1e-5
    assert maxrel(to_np(out["D"]), ref["D"]) <= 1e-4
    assert np.max(np.abs(to_np(out["alpha"]) - ref["scale"])) <= 1e-5
    # the case reaches the clip, and the accumulated-state reading differs from
    # the per-delta one by far more than the tolerance
    assert np.min(ref["scale"]) < 0.9
    per_delta = oracle(cfg, inp)
    assert maxrel(per_delta["D"], ref["D"]) > 1e-2


# The bf16 path: each chunk's V_L^T Z_L from a tcgen05 GEMM, the state kept, clipped
# and copied to bf16 on the CUDA cores.  tau puts some chunks under the clip and
# some over it; the fast-weight term is most of O here, so O sees the scan.
STATE_CLIP_BF16_CASES = {
    # documents inside chunks and at a row's chunk boundary; 128-token chunks, which
    # the per-delta path would scan in groups of 512 tokens
    "bf16_docs": dict(B=2, T=768, C=128, d=256, F=512, eta=2e-2, clip=30.0, docs=[100, 300, 768 + 500]),
    # one document, 256-token chunks: the first unclipped, the rest clipped
    "bf16_tiles": dict(B=1, T=1024, C=256, d=256, F=512, eta=1e-2, clip=30.0, docs=[]),
}


@pytest.mark.parametrize("name", list(STATE_CLIP_BF16_CASES))
def test_state_clip_bf16(name):
    kw = dict(STATE_CLIP_BF16_CASES[name])
    cfg, inp = case(dtype="bf16", conv_std=0.3, wtarget="identity_noise", **kw)
    out = gpu(cfg, inp, state_clip=True)
    ref = state_clip_oracle(cfg, inp)
    errs = (maxrel(to_np(out["O"]), ref["O"]), normrel(to_np(out["S_final"]), ref["S_final"]),
            np.max(np.abs(to_np(out["alpha"]) - ref["scale"])))
    print(name, "O", errs[0], "S_final", errs[1], "clip factors", errs[2])
    assert errs[0] <= 2e-2
    assert errs[1] <= 2e-2
    assert normrel(to_np(out["D"]), ref["D"]) <= 2e-2
    assert errs[2] <= 1e-2
    assert np.min(ref["scale"]) < 0.9 and np.max(ref["scale"]) == 1.0
    per_delta = oracle(cfg, inp)
    assert maxrel(per_delta["O"], ref["O"]) > 5 * 2e-2
