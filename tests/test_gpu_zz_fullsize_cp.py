"""Context-parallel forward at the benchmark's full sizes, ranks emulated in one
process as in test_gpu_cp.py (each rank's begin, the aggregates stacked in rank
order in place of the all-gather, each rank's finish).

Collected after the single-device full-size tests, which hold the single-device
forward at these sizes to the oracle.

Bars:
  * rank 0 sees no incoming state: its outputs are the single-device ones bit for bit;
  * O on every rank within 1e-2 max-relative of the single-device forward (the
    incoming state is added to the bf16 state copies: one more rounding);
  * the last rank's state against the single-device state: both are fp32 sums of the
    same per-chunk deltas (bit-identical: the same MMAs over the same rows), taken
    in another order, so they differ by at most 2 (k-1) u sum_j ||dW_j||_F with
    u = 2^-24; with every delta clipped to tau, sum_j ||dW_j||_F <= k tau;
  * the last rank's state against the fp64 oracle: normwise 2e-2 and no scale bias
    (the bars of the single-device full-size test).
"""
import numpy as np
import pytest
import torch

from chunk_wise_weight_gate_b200 import ipttt as ip
from chunk_wise_weight_gate_b200 import synth
from tests import fullsize_ref
from tests.gpu_util import BIAS_TOL, normrel, scale_bias
from tests.test_gpu_cp import cp_emulated, single

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("name,world", [("qwen3_4b_128k", 8), ("packed_8x8k", 4)])
def test_cp_full_size(name, world):
    w = synth.WORKLOADS[name]
    inp = fullsize_ref.inputs(name)
    cfg = ip.LayerConfig(B=w.B, T=w.T, d=w.d, F=w.F, C=w.C, eta=w.eta, clip=w.clip)
    O, finals = cp_emulated(cfg, inp, world)
    last = finals[-1].cpu()
    del finals
    torch.cuda.empty_cache()
    ref = single(cfg, inp)
    TL = w.T // world
    # compared on the device: bf16 values and their differences are exact in fp32
    Of, Rf = O.float(), ref["O"].float()
    assert torch.isfinite(Of).all()
    assert torch.equal(O[:, :TL], ref["O"][:, :TL])
    assert ((Of - Rf).abs().max() / Rf.abs().max()).item() <= 1e-2
    S_single = ref["S_final"].cpu()
    del O, Of, Rf, ref
    torch.cuda.empty_cache()
    k = w.T // w.C
    b = w.B - 1
    S_ref, _, _ = fullsize_ref.scan_row(name, b)
    x, y = last[b].double().numpy(), S_single[b].double().numpy()
    bound = 2 * (k - 1) * 2.0 ** -24 * k * w.clip / np.linalg.norm(y)
    diff = normrel(x, y)
    print(f"{name}: cp vs single-device state {diff:.3e} (bound {bound:.3e}); "
          f"vs oracle {normrel(x, S_ref):.3e}, scale bias {scale_bias(x, S_ref):+.3e}")
    assert diff <= bound
    assert normrel(x, S_ref) <= 2e-2
    assert abs(scale_bias(x, S_ref)) <= BIAS_TOL
