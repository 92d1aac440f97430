"""Python binding of libipttt.so (the In-Place TTT MLP layer forward on B200).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory and streams.  There is no fallback: if
the shared library is missing, or a tensor is not on a CUDA device, the call
raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# IPTTT_LIB may name another build of the library (for example an instrumented one).
LIB_PATH = os.environ.get("IPTTT_LIB") or os.path.join(_HERE, "libipttt.so")

F32, BF16 = 0, 1
STATUS = {0: "IPTTT_OK", 1: "IPTTT_ERR_ARG", 2: "IPTTT_ERR_SHAPE", 3: "IPTTT_ERR_ALIGN", 4: "IPTTT_ERR_DTYPE",
          5: "IPTTT_ERR_UNSUPPORTED", 6: "IPTTT_ERR_CUDA", 7: "IPTTT_ERR_TIMEOUT", 8: "IPTTT_ERR_WORKSPACE"}
EXPORTS = ("ipttt_workspace_size", "ipttt_forward", "ipttt_forward_ex", "ipttt_core", "ipttt_stream_state_size",
           "ipttt_stream_reset", "ipttt_stream_forward", "ipttt_stream_export", "ipttt_get_status",
           "ipttt_strerror", "ipttt_version", "ipttt_profile_enable", "ipttt_profile_read",
           "ipttt_kernel_launches", "ipttt_selftest_wait_timeout", "ipttt_forward_noalloc",
           "ipttt_forward_host_size", "ipttt_forward_host", "ipttt_decode_state_size", "ipttt_decode_host_size",
           "ipttt_decode_reset", "ipttt_decode_step", "ipttt_decode_export", "ipttt_cp_workspace_size",
           "ipttt_cp_plan", "ipttt_cp_begin", "ipttt_cp_finish", "ipttt_last_error_detail",
           "ipttt_backward_workspace_size", "ipttt_backward")
PHASES = ("prep", "gate_up", "target", "gram", "apply", "update")
DEBUG_OUTPUTS = ("D", "S_final", "alpha", "Z", "V")


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("d", ctypes.c_int32), ("F", ctypes.c_int32),
                ("C", ctypes.c_int32), ("dtype", ctypes.c_int32), ("eta", ctypes.c_float),
                ("clip_thresh", ctypes.c_float), ("flags", ctypes.c_int32)]


FLAG_RESIDUAL = 1
FLAG_STATE_CLIP = 2  # the ablation: clip the accumulated state, not each delta


class IptttError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = last_error_detail() if code == 6 else ""
        super().__init__(f"{where}: {STATUS.get(code, code)} ({strerror(code)})" + (f": {detail}" if detail else ""))


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libipttt.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libipttt.so not built ({LIB_PATH}); run python -m chunk_wise_weight_gate_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, vp, sz, i32 = ctypes.POINTER(Params), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        L.ipttt_workspace_size.argtypes = [P]
        L.ipttt_workspace_size.restype = sz
        L.ipttt_forward.argtypes = [P] + [vp] * 7 + [vp, i32, vp, vp, sz, vp]
        L.ipttt_forward.restype = ctypes.c_int
        L.ipttt_forward_ex.argtypes = [P] + [vp] * 7 + [vp, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.ipttt_forward_ex.restype = ctypes.c_int
        L.ipttt_core.argtypes = [P, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, sz, vp]
        L.ipttt_core.restype = ctypes.c_int
        L.ipttt_stream_state_size.argtypes = [P]
        L.ipttt_stream_state_size.restype = sz
        L.ipttt_stream_reset.argtypes = [P, vp, vp]
        L.ipttt_stream_reset.restype = ctypes.c_int
        L.ipttt_stream_forward.argtypes = [P, vp] + [vp] * 7 + [vp, i32, vp, vp, sz, vp]
        L.ipttt_stream_forward.restype = ctypes.c_int
        L.ipttt_stream_export.argtypes = [P, vp, vp, vp]
        L.ipttt_stream_export.restype = ctypes.c_int
        L.ipttt_get_status.argtypes = [vp]
        L.ipttt_get_status.restype = ctypes.c_int
        L.ipttt_strerror.argtypes = [ctypes.c_int]
        L.ipttt_strerror.restype = ctypes.c_char_p
        L.ipttt_version.argtypes = []
        L.ipttt_version.restype = ctypes.c_char_p
        L.ipttt_last_error_detail.argtypes = []
        L.ipttt_last_error_detail.restype = ctypes.c_char_p
        L.ipttt_backward_workspace_size.argtypes = [P]
        L.ipttt_backward_workspace_size.restype = sz
        L.ipttt_backward.argtypes = [P] + [vp] * 7 + [vp, i32, vp, vp] + [vp] * 7 + [vp, sz, vp]
        L.ipttt_backward.restype = ctypes.c_int
        L.ipttt_profile_enable.argtypes = [ctypes.c_int]
        L.ipttt_profile_enable.restype = None
        L.ipttt_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint64),
                                         ctypes.c_int]
        L.ipttt_profile_read.restype = ctypes.c_int
        L.ipttt_kernel_launches.argtypes = []
        L.ipttt_kernel_launches.restype = ctypes.c_uint64
        L.ipttt_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp]
        L.ipttt_selftest_wait_timeout.restype = ctypes.c_int
        L.ipttt_forward_noalloc.argtypes = [P] + [vp] * 7 + [vp, i32, vp, vp]
        L.ipttt_forward_noalloc.restype = ctypes.c_int
        L.ipttt_forward_host_size.argtypes = [P, i32, i32]
        L.ipttt_forward_host_size.restype = sz
        L.ipttt_forward_host.argtypes = [P] + [vp] * 7 + [vp, i32, vp, vp, sz, i32, vp]
        L.ipttt_forward_host.restype = ctypes.c_int
        L.ipttt_decode_state_size.argtypes = [P]
        L.ipttt_decode_state_size.restype = sz
        L.ipttt_decode_host_size.argtypes = [P]
        L.ipttt_decode_host_size.restype = sz
        L.ipttt_decode_reset.argtypes = [P, vp, vp, vp]
        L.ipttt_decode_reset.restype = ctypes.c_int
        L.ipttt_decode_step.argtypes = [P, vp, vp, vp, vp, vp] + [vp] * 5 + [vp, vp]
        L.ipttt_decode_step.restype = ctypes.c_int
        L.ipttt_decode_export.argtypes = [P, vp, vp, vp]
        L.ipttt_decode_export.restype = ctypes.c_int
        L.ipttt_cp_workspace_size.argtypes = [P]
        L.ipttt_cp_workspace_size.restype = sz
        L.ipttt_cp_plan.argtypes = [P, i32, i32, vp, i32, vp, vp, vp]
        L.ipttt_cp_plan.restype = ctypes.c_int
        L.ipttt_cp_begin.argtypes = [P, i32, i32, vp, i32] + [vp] * 6 + [vp, vp, sz, vp]
        L.ipttt_cp_begin.restype = ctypes.c_int
        L.ipttt_cp_finish.argtypes = [P, i32, i32, vp, i32, vp, vp, vp, vp, vp, vp, sz, vp]
        L.ipttt_cp_finish.restype = ctypes.c_int
        _lib = L
    return _lib


def strerror(code: int) -> str:
    try:
        return lib().ipttt_strerror(code).decode()
    except Exception:  # library missing while formatting an error
        return "?"


def last_error_detail() -> str:
    """The CUDA error behind this thread's last IPTTT_ERR_CUDA ("" if none)."""
    try:
        return lib().ipttt_last_error_detail().decode()
    except Exception:
        return ""


def _check(code: int, where: str):
    if code != 0:
        raise IptttError(code, where)


@dataclass
class LayerConfig:
    B: int
    T: int
    d: int
    F: int
    C: int
    eta: float
    clip: float = 0.0
    dtype: str = "bf16"

    def params(self, flags: int = 0) -> Params:
        return Params(self.B, self.T, self.d, self.F, self.C, BF16 if self.dtype == "bf16" else F32,
                      float(self.eta), float(self.clip), int(flags))

    @property
    def k(self) -> int:
        return (self.T + self.C - 1) // self.C

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor") -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _docs(doc_starts, device) -> tuple[int | None, int, torch.Tensor | None]:
    if doc_starts is None:
        return None, 0, None
    ds = doc_starts if isinstance(doc_starts, torch.Tensor) else torch.as_tensor(doc_starts, dtype=torch.int32)
    ds = ds.to(device=device, dtype=torch.int32).contiguous()
    if ds.numel() == 0:
        return None, 0, ds
    return ds.data_ptr(), int(ds.numel()), ds


def workspace_size(cfg: LayerConfig, state_clip: bool = False) -> int:
    """Workspace bytes of a forward (state_clip: of the accumulated-state clip, which
    keeps each chunk's raw delta in fp32 on the bf16 path too)."""
    n = lib().ipttt_workspace_size(ctypes.byref(cfg.params(FLAG_STATE_CLIP if state_clip else 0)))
    if n == 0:
        raise ValueError(f"invalid layer configuration {cfg}")
    return int(n)


def alloc_workspace(cfg: LayerConfig, device="cuda", state_clip: bool = False) -> torch.Tensor:
    return torch.empty(workspace_size(cfg, state_clip), dtype=torch.uint8, device=device)


def _shape_check(cfg: LayerConfig, **tensors):
    want = {"H": (cfg.B, cfg.T, cfg.d), "X0": (cfg.B, cfg.T, cfg.d), "Wgate": (cfg.F, cfg.d),
            "Wup": (cfg.F, cfg.d), "Wdown0": (cfg.d, cfg.F), "conv_w": (cfg.d, 5), "Wtarget": (cfg.d, cfg.d),
            "Z": (cfg.B, cfg.T, cfg.F), "V": (cfg.B, cfg.T, cfg.d), "O": (cfg.B, cfg.T, cfg.d)}
    for name, t in tensors.items():
        if t is not None and tuple(t.shape) != want[name]:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want[name]}")


def forward(cfg: LayerConfig, H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, doc_starts=None, *, O=None,
            workspace=None, stream=None, debug=False, residual=False, state_clip=False):
    """One layer forward.  Returns O, or with debug=True (or a subset of
    DEBUG_OUTPUTS) a dict with O and the chosen internals D, S_final, alpha, Z, V,
    produced by the same kernels as O.  residual=True writes H + output into O.
    state_clip=True clips the accumulated state instead of each delta; alpha then
    holds the state's clip factor per chunk."""
    dt = cfg.torch_dtype
    _shape_check(cfg, H=H, X0=X0, Wgate=Wgate, Wup=Wup, Wdown0=Wdown0, conv_w=conv_w, Wtarget=Wtarget, O=O)
    dev = H.device
    if O is None:
        O = torch.empty(cfg.B, cfg.T, cfg.d, dtype=dt, device=dev)
    if workspace is None:
        workspace = alloc_workspace(cfg, dev, state_clip)
    if residual and O.data_ptr() == H.data_ptr():
        raise ValueError("O must not alias H when residual=True")
    dp, nd, keep = _docs(doc_starts, dev)
    p = cfg.params((FLAG_RESIDUAL if residual else 0) | (FLAG_STATE_CLIP if state_clip else 0))
    args = [_ptr(H, dt, "H"), _ptr(X0, dt, "X0"), _ptr(Wgate, dt, "Wgate"), _ptr(Wup, dt, "Wup"),
            _ptr(Wdown0, dt, "Wdown0"), _ptr(conv_w, dt, "conv_w"), _ptr(Wtarget, dt, "Wtarget"), dp, nd,
            _ptr(O, dt, "O")]
    if not debug:
        _check(lib().ipttt_forward(ctypes.byref(p), *args, workspace.data_ptr(), workspace.numel(),
                                   _stream(stream)), "ipttt_forward")
        return O
    want = set(DEBUG_OUTPUTS) if debug is True else set(debug)
    shapes = {"D": ((cfg.B, cfg.T, cfg.d), torch.float32), "S_final": ((cfg.B, cfg.d, cfg.F), torch.float32),
              "alpha": ((cfg.B, cfg.k), torch.float32), "Z": ((cfg.B, cfg.T, cfg.F), dt),
              "V": ((cfg.B, cfg.T, cfg.d), dt)}
    out = {"O": O}
    for name in DEBUG_OUTPUTS:
        out[name] = torch.empty(*shapes[name][0], dtype=shapes[name][1], device=dev) if name in want else None
    ptrs = [out[n].data_ptr() if out[n] is not None else None for n in DEBUG_OUTPUTS]
    _check(lib().ipttt_forward_ex(ctypes.byref(p), *args, *ptrs, workspace.data_ptr(), workspace.numel(),
                                  _stream(stream)), "ipttt_forward_ex")
    return out


def core(cfg: LayerConfig, Z, V, Wdown0, doc_starts=None, *, workspace=None, stream=None):
    """The chunk scan alone on given Z [B,T,F] and V [B,T,d]; returns O, D, S_final, alpha."""
    dt = cfg.torch_dtype
    _shape_check(cfg, Z=Z, V=V, Wdown0=Wdown0)
    dev = Z.device
    if workspace is None:
        workspace = alloc_workspace(cfg, dev)
    dp, nd, keep = _docs(doc_starts, dev)
    out = {"O": torch.empty(cfg.B, cfg.T, cfg.d, dtype=dt, device=dev),
           "D": torch.empty(cfg.B, cfg.T, cfg.d, dtype=torch.float32, device=dev),
           "S_final": torch.empty(cfg.B, cfg.d, cfg.F, dtype=torch.float32, device=dev),
           "alpha": torch.empty(cfg.B, cfg.k, dtype=torch.float32, device=dev)}
    p = cfg.params()
    _check(lib().ipttt_core(ctypes.byref(p), _ptr(Z, dt, "Z"), _ptr(V, dt, "V"), _ptr(Wdown0, dt, "Wdown0"), dp,
                            nd, out["O"].data_ptr(), out["D"].data_ptr(), out["S_final"].data_ptr(),
                            out["alpha"].data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "ipttt_core")
    return out


def backward_workspace_size(cfg: LayerConfig) -> int:
    """Bytes of device workspace ipttt_backward needs for this configuration."""
    p = cfg.params()
    n = lib().ipttt_backward_workspace_size(ctypes.byref(p))
    if n == 0:
        raise ValueError(f"invalid layer configuration {cfg}")
    return n


def backward(cfg: LayerConfig, H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, doc_starts, gO, gS_final=None, *,
             workspace=None, stream=None):
    """fp32 gradients of <gO, O> + <gS_final, S_final> with respect to the layer's
    inputs (ipttt_backward); returns a dict keyed like the inputs."""
    dt = cfg.torch_dtype
    _shape_check(cfg, H=H, X0=X0, Wgate=Wgate, Wup=Wup, Wdown0=Wdown0, conv_w=conv_w, Wtarget=Wtarget, O=gO)
    dev = H.device
    p = cfg.params()
    if workspace is None:
        workspace = torch.empty(backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    f32 = torch.float32
    out = {"H": torch.empty(cfg.B, cfg.T, cfg.d, dtype=f32, device=dev),
           "X0": torch.empty(cfg.B, cfg.T, cfg.d, dtype=f32, device=dev),
           "Wgate": torch.empty(cfg.F, cfg.d, dtype=f32, device=dev),
           "Wup": torch.empty(cfg.F, cfg.d, dtype=f32, device=dev),
           "Wdown0": torch.empty(cfg.d, cfg.F, dtype=f32, device=dev),
           "conv_w": torch.empty(cfg.d, 5, dtype=f32, device=dev),
           "Wtarget": torch.empty(cfg.d, cfg.d, dtype=f32, device=dev)}
    if gS_final is not None and tuple(gS_final.shape) != (cfg.B, cfg.d, cfg.F):
        raise ValueError(f"gS_final has shape {tuple(gS_final.shape)}, expected {(cfg.B, cfg.d, cfg.F)}")
    dp, nd, keep = _docs(doc_starts, dev)
    _check(lib().ipttt_backward(ctypes.byref(p), _ptr(H, dt, "H"), _ptr(X0, dt, "X0"), _ptr(Wgate, dt, "Wgate"),
                                _ptr(Wup, dt, "Wup"), _ptr(Wdown0, dt, "Wdown0"), _ptr(conv_w, dt, "conv_w"),
                                _ptr(Wtarget, dt, "Wtarget"), dp, nd, _ptr(gO, dt, "gO"),
                                _ptr(gS_final, f32, "gS_final"),
                                *(out[k].data_ptr() for k in ("H", "X0", "Wgate", "Wup", "Wdown0", "conv_w",
                                                             "Wtarget")),
                                workspace.data_ptr(), workspace.numel(), _stream(stream)), "ipttt_backward")
    return out


def forward_host_size(cfg: LayerConfig, piece_tokens: int = 0, n_doc_starts: int = 0) -> int:
    """Device bytes ipttt_forward_host needs (0 for an invalid piece length)."""
    return int(lib().ipttt_forward_host_size(ctypes.byref(cfg.params()), piece_tokens, n_doc_starts))


def _host_ptr(t: torch.Tensor, dtype, name: str) -> int:
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def forward_host(cfg: LayerConfig, H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, doc_starts=None, *, O=None,
                 piece_tokens: int = 0, buffer=None, stream=None):
    """One layer forward with H, X0 and O in host memory (page-locked tensors let
    the copies overlap the compute) and the weights on the device; the sequence is
    pipelined through the streaming path in pieces of piece_tokens tokens (0: about
    T/8).  Returns O, a host tensor that is complete once `stream` has finished."""
    dt = cfg.torch_dtype
    for name, t in (("H", H), ("X0", X0)):
        if tuple(t.shape) != (cfg.B, cfg.T, cfg.d):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {(cfg.B, cfg.T, cfg.d)}")
    _shape_check(cfg, Wgate=Wgate, Wup=Wup, Wdown0=Wdown0, conv_w=conv_w, Wtarget=Wtarget)
    dev = Wgate.device
    if O is None:
        O = torch.empty(cfg.B, cfg.T, cfg.d, dtype=dt, pin_memory=H.is_pinned())
    ds = None
    if doc_starts is not None:
        ds = doc_starts if isinstance(doc_starts, torch.Tensor) else torch.as_tensor(doc_starts, dtype=torch.int32)
        ds = ds.to(device="cpu", dtype=torch.int32).contiguous()
    nd = 0 if ds is None else ds.numel()
    need = forward_host_size(cfg, piece_tokens, nd)
    if need == 0:
        raise ValueError(f"invalid piece length {piece_tokens} for chunk {cfg.C}")
    if buffer is None:
        buffer = torch.empty(need, dtype=torch.uint8, device=dev)
    p = cfg.params()
    _check(lib().ipttt_forward_host(ctypes.byref(p), _host_ptr(H, dt, "H"), _host_ptr(X0, dt, "X0"),
                                    _ptr(Wgate, dt, "Wgate"), _ptr(Wup, dt, "Wup"), _ptr(Wdown0, dt, "Wdown0"),
                                    _ptr(conv_w, dt, "conv_w"), _ptr(Wtarget, dt, "Wtarget"),
                                    ds.data_ptr() if nd else None, nd, _host_ptr(O, dt, "O"), buffer.data_ptr(),
                                    buffer.numel(), piece_tokens, _stream(stream)), "ipttt_forward_host")
    return O


# ---------------------------------------------------------------- context parallelism
# cfg.T is the shard length: rank r of `world` holds tokens [r*T, (r+1)*T) of every
# row; doc_starts are offsets b*(world*T) + t over the whole sequence, on the host.

def _host_docs(doc_starts) -> torch.Tensor:
    if doc_starts is None:
        return torch.zeros(0, dtype=torch.int32)
    ds = doc_starts if isinstance(doc_starts, torch.Tensor) else torch.as_tensor(doc_starts, dtype=torch.int32)
    return ds.to(device="cpu", dtype=torch.int32).contiguous()


def cp_workspace_size(cfg: LayerConfig) -> int:
    n = lib().ipttt_cp_workspace_size(ctypes.byref(cfg.params()))
    if n == 0:
        raise ValueError(f"invalid context-parallel configuration {cfg}")
    return int(n)


def cp_plan(cfg: LayerConfig, world: int, rank: int, doc_starts=None):
    """Host side of the split (no GPU needed): this rank's document starts as
    offsets within the shard, and the per-row plan dict (row_cont, first_rank,
    prefix_chunks, keep), each a list of B ints."""
    ds = _host_docs(doc_starts)
    nd = ds.numel()
    local = torch.zeros(max(nd, 1), dtype=torch.int32)
    plan = torch.zeros(4, cfg.B, dtype=torch.int32)
    n_local = ctypes.c_int32(0)
    p = cfg.params()
    _check(lib().ipttt_cp_plan(ctypes.byref(p), int(world), int(rank), ds.data_ptr() if nd else None, nd,
                               local.data_ptr(), ctypes.addressof(n_local), plan.data_ptr()), "ipttt_cp_plan")
    names = ("row_cont", "first_rank", "prefix_chunks", "keep")
    return local[:n_local.value].tolist(), {n: plan[i].tolist() for i, n in enumerate(names)}


def cp_begin(cfg: LayerConfig, world: int, rank: int, H, X0, Wgate, Wup, conv_w, Wtarget, doc_starts=None, *,
             agg=None, workspace=None, stream=None):
    """First stage on one rank: the shard's forward up to its state updates.
    Returns (agg, workspace); agg [B, d, F] fp32 is what the ranks exchange, and
    the workspace goes unchanged to cp_finish."""
    dt = cfg.torch_dtype
    _shape_check(cfg, H=H, X0=X0, Wgate=Wgate, Wup=Wup, conv_w=conv_w, Wtarget=Wtarget)
    dev = H.device
    if agg is None:
        agg = torch.empty(cfg.B, cfg.d, cfg.F, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(cp_workspace_size(cfg), dtype=torch.uint8, device=dev)
    ds = _host_docs(doc_starts)
    nd = ds.numel()
    p = cfg.params()
    _check(lib().ipttt_cp_begin(ctypes.byref(p), int(world), int(rank), ds.data_ptr() if nd else None, nd,
                                _ptr(H, dt, "H"), _ptr(X0, dt, "X0"), _ptr(Wgate, dt, "Wgate"), _ptr(Wup, dt, "Wup"),
                                _ptr(conv_w, dt, "conv_w"), _ptr(Wtarget, dt, "Wtarget"),
                                _ptr(agg, torch.float32, "agg"), workspace.data_ptr(), workspace.numel(),
                                _stream(stream)), "ipttt_cp_begin")
    return agg, workspace


def cp_exchange(agg: torch.Tensor, group=None, out: torch.Tensor | None = None) -> torch.Tensor:
    """The one exchange: every rank's aggregate, gathered in rank order
    ([world, B, d, F]; into `out` when given), through torch.distributed (NCCL on
    GPUs)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if out is None:
        out = torch.empty(world, *agg.shape, dtype=agg.dtype, device=agg.device)
    if tuple(out.shape) != (world, *agg.shape) or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {(world, *agg.shape)} tensor")
    dist.all_gather_into_tensor(out.view(-1), agg.contiguous().view(-1), group=group)
    return out


def cp_finish(cfg: LayerConfig, world: int, rank: int, H, Wdown0, gathered, workspace, doc_starts=None, *, O=None,
              S_final=False, residual=False, stream=None):
    """Second stage on one rank: returns this shard's O (and S_final, the state
    after the shard's last chunk, when S_final=True)."""
    dt = cfg.torch_dtype
    _shape_check(cfg, H=H, Wdown0=Wdown0, O=O)
    if tuple(gathered.shape) != (world, cfg.B, cfg.d, cfg.F):
        raise ValueError(f"gathered has shape {tuple(gathered.shape)}, expected {(world, cfg.B, cfg.d, cfg.F)}")
    dev = H.device
    if O is None:
        O = torch.empty(cfg.B, cfg.T, cfg.d, dtype=dt, device=dev)
    if residual and O.data_ptr() == H.data_ptr():
        raise ValueError("O must not alias H when residual=True")
    Sf = torch.empty(cfg.B, cfg.d, cfg.F, dtype=torch.float32, device=dev) if S_final else None
    ds = _host_docs(doc_starts)
    nd = ds.numel()
    p = cfg.params(FLAG_RESIDUAL if residual else 0)
    _check(lib().ipttt_cp_finish(ctypes.byref(p), int(world), int(rank), ds.data_ptr() if nd else None, nd,
                                 _ptr(H, dt, "H"), _ptr(Wdown0, dt, "Wdown0"),
                                 _ptr(gathered, torch.float32, "gathered"), _ptr(O, dt, "O"),
                                 Sf.data_ptr() if Sf is not None else None, workspace.data_ptr(), workspace.numel(),
                                 _stream(stream)), "ipttt_cp_finish")
    return (O, Sf) if S_final else O


def cp_forward(cfg: LayerConfig, H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, doc_starts=None, *, group=None,
               S_final=False, residual=False, stream=None):
    """This rank's shard of a context-parallel forward over the ranks of `group`:
    begin, one all-gather of the shard aggregates, finish."""
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    agg, ws = cp_begin(cfg, world, rank, H, X0, Wgate, Wup, conv_w, Wtarget, doc_starts, stream=stream)
    gathered = cp_exchange(agg, group)
    return cp_finish(cfg, world, rank, H, Wdown0, gathered, ws, doc_starts, S_final=S_final, residual=residual,
                     stream=stream)


class StreamState:
    """Caller-owned fast-weight state carried between pieces of long sequences."""

    def __init__(self, cfg: LayerConfig, device="cuda", stream=None):
        self.cfg = cfg
        n = lib().ipttt_stream_state_size(ctypes.byref(cfg.params()))
        if n == 0:
            raise ValueError(f"invalid layer configuration {cfg}")
        self.buf = torch.empty(int(n), dtype=torch.uint8, device=device)
        self.reset(stream)

    def reset(self, stream=None):
        _check(lib().ipttt_stream_reset(ctypes.byref(self.cfg.params()), self.buf.data_ptr(), _stream(stream)),
               "ipttt_stream_reset")

    def forward(self, piece_cfg: LayerConfig, H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, doc_starts=None, *,
                workspace=None, stream=None):
        dt = piece_cfg.torch_dtype
        _shape_check(piece_cfg, H=H, X0=X0)
        dev = H.device
        O = torch.empty(piece_cfg.B, piece_cfg.T, piece_cfg.d, dtype=dt, device=dev)
        if workspace is None:
            workspace = alloc_workspace(piece_cfg, dev)
        dp, nd, keep = _docs(doc_starts, dev)
        p = piece_cfg.params()
        _check(lib().ipttt_stream_forward(ctypes.byref(p), self.buf.data_ptr(), _ptr(H, dt, "H"),
                                          _ptr(X0, dt, "X0"), _ptr(Wgate, dt, "Wgate"), _ptr(Wup, dt, "Wup"),
                                          _ptr(Wdown0, dt, "Wdown0"), _ptr(conv_w, dt, "conv_w"),
                                          _ptr(Wtarget, dt, "Wtarget"), dp, nd, O.data_ptr(),
                                          workspace.data_ptr(), workspace.numel(), _stream(stream)),
               "ipttt_stream_forward")
        return O

    def export(self, stream=None) -> torch.Tensor:
        S = torch.empty(self.cfg.B, self.cfg.d, self.cfg.F, dtype=torch.float32, device=self.buf.device)
        _check(lib().ipttt_stream_export(ctypes.byref(self.cfg.params()), self.buf.data_ptr(), S.data_ptr(),
                                         _stream(stream)), "ipttt_stream_export")
        return S


class DecodeState:
    """Token-by-token decoding of B rows (bf16, B <= 16): a device state buffer and
    the host bookkeeping the library keeps between steps.  cfg.T is ignored."""

    def __init__(self, cfg: LayerConfig, device="cuda", stream=None):
        self.cfg = cfg
        p = cfg.params()
        n = int(lib().ipttt_decode_state_size(ctypes.byref(p)))
        nh = int(lib().ipttt_decode_host_size(ctypes.byref(p)))
        if n == 0 or nh == 0:
            raise ValueError("decoding needs bf16 and at most 16 rows")
        self.buf = torch.empty(n, dtype=torch.uint8, device=device)
        self.host = ctypes.create_string_buffer(nh)
        self.reset(stream)

    def reset(self, stream=None):
        _check(lib().ipttt_decode_reset(ctypes.byref(self.cfg.params()), self.buf.data_ptr(), self.host,
                                        _stream(stream)), "ipttt_decode_reset")

    def step(self, h, x0, Wgate, Wup, Wdown0, conv_w, Wtarget, starts=None, *, o=None, stream=None):
        """One token of every row: h, x0 [B, d] on the device; starts: B flags (a
        document begins at this token), or None.  Returns o [B, d].  The weights
        are checked once per set of tensors (by identity) and their pointers kept."""
        cfg = self.cfg
        dt = cfg.torch_dtype
        for name, t in (("h", h), ("x0", x0)):
            if tuple(t.shape) != (cfg.B, cfg.d):
                raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {(cfg.B, cfg.d)}")
        ws = (Wgate, Wup, Wdown0, conv_w, Wtarget)
        key = tuple(id(w) for w in ws)
        if getattr(self, "_wkey", None) != key:
            _shape_check(cfg, Wgate=Wgate, Wup=Wup, Wdown0=Wdown0, conv_w=conv_w, Wtarget=Wtarget)
            self._wptr = [_ptr(w, dt, n) for w, n in zip(ws, ("Wgate", "Wup", "Wdown0", "conv_w", "Wtarget"))]
            self._wref = ws  # keeps the tensors (and so their ids and pointers) alive
            self._wkey = key
        if getattr(self, "_p", None) is None:
            self._p = cfg.params()
        if o is None:
            o = torch.empty(cfg.B, cfg.d, dtype=dt, device=h.device)
        flags = None
        if starts is not None:
            flags = (ctypes.c_int32 * cfg.B)(*[int(bool(x)) for x in starts])
        _check(lib().ipttt_decode_step(ctypes.byref(self._p), self.buf.data_ptr(), self.host,
                                       _ptr(h, dt, "h"), _ptr(x0, dt, "x0"), flags, *self._wptr, _ptr(o, dt, "o"),
                                       _stream(stream)),
               "ipttt_decode_step")
        return o

    def export(self, stream=None) -> torch.Tensor:
        """The committed fp32 state [B, d, F]."""
        S = torch.empty(self.cfg.B, self.cfg.d, self.cfg.F, dtype=torch.float32, device=self.buf.device)
        _check(lib().ipttt_decode_export(ctypes.byref(self.cfg.params()), self.buf.data_ptr(), S.data_ptr(),
                                         _stream(stream)), "ipttt_decode_export")
        return S


def get_status(stream=None) -> int:
    """Waits for the stream and returns (and clears) the device status word."""
    return int(lib().ipttt_get_status(_stream(stream)))


def profile_enable(on: bool = True):
    lib().ipttt_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """Per phase: (milliseconds, kernel launches) accumulated since the last read."""
    n = len(PHASES)
    ms = (ctypes.c_double * n)()
    ln = (ctypes.c_uint64 * n)()
    lib().ipttt_profile_read(ms, ln, n)
    return {PHASES[i]: (float(ms[i]), int(ln[i])) for i in range(n)}


def selftest_wait_timeout(limit_ns: int = 100_000_000, stream=None):
    """Runs the bounded-wait failure path on the device (see include/ipttt.h)."""
    _check(lib().ipttt_selftest_wait_timeout(int(limit_ns), _stream(stream)), "ipttt_selftest_wait_timeout")


def kernel_launches() -> int:
    return int(lib().ipttt_kernel_launches())


def version() -> str:
    return lib().ipttt_version().decode()


def flops_per_token(d: int, F: int) -> int:
    """Credited flops per token: gate/up 4dF, Z W0^T 2dF, Z S^T 2dF, delta 2dF,
    target projection 2d^2, conv 10d (the Gram pass for the clip is not credited)."""
    return 10 * d * F + 2 * d * d + 10 * d


def chunks(T: int, C: int) -> int:
    return math.ceil(T / C)
