"""Seeded synthetic workloads for the In-Place TTT MLP layer.

This module only draws numbers: it holds none of the layer's arithmetic, so the
CUDA path and the fp64 oracle can both be fed from it without sharing any code
of the method.  Every tensor comes from numpy's counter-based Philox generator,
keyed by (seed, layer, tensor id, row block), so a tensor's values do not depend
on how many threads draw it or on which other tensors are drawn.

Distributions follow the workload descriptions of the layer's headline
configurations (Qwen3-4B MLP shape d_model=2560, d_ff=9728):

* H, X0 ~ N(0, 1)
* Wgate, Wup ~ N(0, 1/d) and Wdown0 ~ N(0, 1/d_ff)  (variance 1/fan_in)
* depthwise conv taps [d, 5] ~ N(0, std) with std 0.1 (tiny fp32 case) or 0.02
* Wtarget: identity + dense N(0, 0.01) noise (tiny case), or sparse-diagonal:
  diagonal ~ N(1, 0.05), 1% of off-diagonal entries ~ N(0, 0.01), the rest 0
* packed documents: lengths ~ U{256..4096}, cut at the row length T

A second argument of N(mu, x) given as a literal (0.1, 0.05, 0.02, 0.01) is a
standard deviation; "1/fan_in" is a variance.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

_TENSOR_IDS = {"H": 1, "X0": 2, "Wgate": 3, "Wup": 4, "Wdown0": 5, "conv_w": 6,
               "Wtarget": 7, "Wtarget_mask": 8, "Wtarget_off": 9, "docs": 10}
_ROWS_PER_BLOCK = 4096


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    C: int
    d: int
    F: int
    dtype: str = "bf16"          # "f32" or "bf16": storage and operand type
    eta: float = 1e-3
    clip: float = 1e-5           # <= 0 means no clip
    docs: str = "single"         # "single" or "packed"
    conv_std: float = 0.02
    wtarget: str = "sparse_diag"  # "sparse_diag" or "identity_noise"
    layers: int = 1

    @property
    def tokens(self) -> int:
        return self.B * self.T * self.layers

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five headline configurations of the layer.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", B=1, T=256, C=32, d=64, F=256, dtype="f32",
                         eta=0.01, clip=0.0, conv_std=0.1, wtarget="identity_noise"),
    "qwen3_4b_32k": Workload("qwen3_4b_32k", B=1, T=32768, C=512, d=2560, F=9728),
    "qwen3_4b_128k": Workload("qwen3_4b_128k", B=1, T=131072, C=1024, d=2560, F=9728),
    "packed_8x8k": Workload("packed_8x8k", B=8, T=8192, C=512, d=2560, F=9728, docs="packed"),
    "stack6_4x16k": Workload("stack6_4x16k", B=4, T=16384, C=512, d=2560, F=9728, layers=6),
    # the Qwen3-4B layer on 4k tokens: a small case for profiler captures
    "qwen3_4b_4k": Workload("qwen3_4b_4k", B=1, T=4096, C=512, d=2560, F=9728),
}
STACK_CHUNK_SIZES = (64, 128, 256, 512, 1024, 2048)


def _philox(seed: int, layer: int, tensor: str, block: int) -> np.random.Generator:
    key = [(int(seed) & 0xFFFFFFFF) << 32 | (int(layer) & 0xFFFF) << 16 | _TENSOR_IDS[tensor],
           int(block)]
    return np.random.Generator(np.random.Philox(key=key))


def _normal_rows(shape, mean, std, seed, layer, tensor, threads=8) -> np.ndarray:
    """N(mean, std^2) float32 array; rows drawn in fixed blocks, each block its own key."""
    rows = shape[0]
    inner = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    out = np.empty((rows, inner), dtype=np.float32)

    def fill(blk):
        r0 = blk * _ROWS_PER_BLOCK
        r1 = min(rows, r0 + _ROWS_PER_BLOCK)
        g = _philox(seed, layer, tensor, blk)
        out[r0:r1] = g.standard_normal((r1 - r0, inner), dtype=np.float32)

    nblk = (rows + _ROWS_PER_BLOCK - 1) // _ROWS_PER_BLOCK
    if nblk > 1 and threads > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(nblk)))
    else:
        for b in range(nblk):
            fill(b)
    if std != 1.0:
        out *= np.float32(std)
    if mean != 0.0:
        out += np.float32(mean)
    return out.reshape(shape)


def doc_starts_for(w: Workload, seed: int = 0) -> np.ndarray:
    """Sorted global offsets b*T + t of document starts that are not row starts."""
    if w.docs == "single":
        return np.zeros((0,), dtype=np.int32)
    starts = []
    for b in range(w.B):
        g = _philox(seed, 0, "docs", b)
        t = 0
        while True:
            t += int(g.integers(256, 4097))
            if t >= w.T:
                break
            starts.append(b * w.T + t)
    return np.asarray(starts, dtype=np.int32)


def _to(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.bfloat16) if dtype == "bf16" else t.to(torch.float32)


def make_inputs(w: Workload, seed: int = 0, layer: int = 0, with_activations: bool = True):
    """Draw one layer's inputs as CPU tensors in the workload's dtype.

    Returns a dict with H, X0 [B,T,d]; Wgate, Wup [F,d]; Wdown0 [d,F]; conv_w [d,5];
    Wtarget [d,d]; doc_starts (int32, global offsets, row starts implicit).
    """
    d, F = w.d, w.F
    out = {}
    if with_activations:
        out["H"] = _to(_normal_rows((w.B * w.T, d), 0.0, 1.0, seed, layer, "H"), w.dtype).view(w.B, w.T, d)
        out["X0"] = _to(_normal_rows((w.B * w.T, d), 0.0, 1.0, seed, 0, "X0"), w.dtype).view(w.B, w.T, d)
    out["Wgate"] = _to(_normal_rows((F, d), 0.0, d ** -0.5, seed, layer, "Wgate"), w.dtype)
    out["Wup"] = _to(_normal_rows((F, d), 0.0, d ** -0.5, seed, layer, "Wup"), w.dtype)
    out["Wdown0"] = _to(_normal_rows((d, F), 0.0, F ** -0.5, seed, layer, "Wdown0"), w.dtype)
    out["conv_w"] = _to(_normal_rows((d, 5), 0.0, w.conv_std, seed, layer, "conv_w"), w.dtype)
    if w.wtarget == "identity_noise":
        wt = _normal_rows((d, d), 0.0, 0.01, seed, layer, "Wtarget")
        wt += np.eye(d, dtype=np.float32)
    else:
        diag = _normal_rows((d, 1), 1.0, 0.05, seed, layer, "Wtarget")[:, 0]
        g = _philox(seed, layer, "Wtarget_mask", 0)
        mask = g.random((d, d)) < 0.01
        off = _normal_rows((d, d), 0.0, 0.01, seed, layer, "Wtarget_off")
        wt = np.where(mask, off, np.float32(0.0)).astype(np.float32)
        np.fill_diagonal(wt, diag)
    out["Wtarget"] = _to(wt, w.dtype)
    out["doc_starts"] = torch.from_numpy(doc_starts_for(w, seed))
    return out


def random_doc_starts(B: int, T: int, n_per_row: int, seed: int, min_gap: int = 1) -> np.ndarray:
    """Uniformly placed document starts (global offsets) for small test cases."""
    g = _philox(seed, 0, "docs", 1 << 20)
    starts = []
    for b in range(B):
        cand = np.arange(min_gap, T)
        k = min(n_per_row, len(cand))
        pick = np.sort(g.choice(cand, size=k, replace=False)) if k > 0 else []
        starts.extend(int(b * T + p) for p in pick)
    return np.asarray(starts, dtype=np.int32)
