"""The objective ablations of cloud.tencent.com "榨干MLP的剩余价值", 验证模块三
(目标组件剥离) and the admirer.cn article, 五: the LM-aligned target without its
conv or without its projection.  Both are weight settings of the unchanged layer,
so they run through the same kernels and are held to the same bars as every bf16
parity case (oracle/ipttt_ablations.py gives the weights)."""
import numpy as np
import pytest
import torch

from oracle import ipttt_ablations as ab
from tests.gpu_util import case, gpu, oracle, to_np
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
