"""Host-side checks of libipttt.so that need no GPU: it loads, exports every
symbol that include/ipttt.h declares, and rejects bad arguments before any
CUDA call."""
import ctypes
import os
import re

import pytest

from chunk_wise_weight_gate_b200 import ipttt as ip

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "ipttt.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"IPTTT_API\s+[\w\s\*]+?\b(ipttt_\w+)\s*\(", text)))


def test_header_declares_the_expected_entry_points():
    assert declared_functions() == sorted(ip.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = ip.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def test_version_and_strerror():
    assert re.fullmatch(r"\d+\.\d+\.\d+", ip.version())
    for code in range(9):
        assert ip.strerror(code) not in ("", "unknown status")
    assert ip.strerror(99) == "unknown status"


def params(**kw):
    base = dict(B=1, T=512, d=256, F=512, C=128, dtype=ip.BF16, eta=1e-3, clip_thresh=1e-5, flags=0)
    base.update(kw)
    return ip.Params(**base)


def call_forward(p, ptrs=None, ws=0x100000, ws_bytes=None, n_doc=0, doc=None):
    L = ip.lib()
    fake = ptrs or [0x10000 + 256 * i for i in range(8)]
    if ws_bytes is None:
        ws_bytes = L.ipttt_workspace_size(ctypes.byref(p))
    return L.ipttt_forward(ctypes.byref(p), *fake[:7], doc, n_doc, fake[7], ws, ws_bytes, None)


def test_workspace_size_grows_with_tokens_and_is_zero_when_invalid():
    L = ip.lib()
    a = L.ipttt_workspace_size(ctypes.byref(params()))
    b = L.ipttt_workspace_size(ctypes.byref(params(T=1024)))
    assert 0 < a < b
    assert a % 256 == 0
    assert L.ipttt_workspace_size(ctypes.byref(params(B=0))) == 0
    assert L.ipttt_workspace_size(ctypes.byref(params(dtype=7))) == 0
    # The bf16 workspace holds Z (bf16 [B,T,F]) at least.
    assert a >= 512 * 512 * 2


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), 1), (dict(T=-1), 1), (dict(C=0), 1), (dict(dtype=3), 4),
    (dict(eta=float("nan")), 1), (dict(clip_thresh=float("nan")), 1),
    (dict(d=200), 5), (dict(F=320), 5), (dict(C=96), 5), (dict(C=32), 5), (dict(C=8192), 5), (dict(flags=6), 1),
])
def test_bad_params_are_rejected_before_launch(kw, code):
    assert call_forward(params(**kw)) == code


def test_state_clip_only_where_it_has_a_meaning():
    # the forward takes the accumulated-state clip on both paths, with room for the
    # raw delta; the backward (its gradients are those of the per-delta clip) and
    # the context-parallel split (the clip is not linear in the state) do not
    L = ip.lib()
    for dt in (ip.BF16, ip.F32):
        plain = L.ipttt_workspace_size(ctypes.byref(params(dtype=dt)))
        clip = L.ipttt_workspace_size(ctypes.byref(params(dtype=dt, flags=2)))
        assert clip >= plain > 0
        assert L.ipttt_backward_workspace_size(ctypes.byref(params(dtype=dt, flags=2))) == 0
        assert L.ipttt_backward_workspace_size(ctypes.byref(params(dtype=dt))) > 0
    assert L.ipttt_decode_state_size(ctypes.byref(params(flags=2))) == 0
    p = params(flags=2)
    fake = [0x10000 + 256 * i for i in range(8)]
    rc = L.ipttt_cp_begin(ctypes.byref(p), 2, 0, None, 0, *fake[:6], ctypes.c_void_p(fake[6]),
                          ctypes.c_void_p(0x100000), ctypes.c_size_t(1 << 40), None)
    assert rc == 5


def test_null_misaligned_and_workspace_errors():
    p = params()
    ptrs = [0x10000 + 256 * i for i in range(8)]
    bad = list(ptrs); bad[0] = 0
    assert call_forward(p, bad) == 1                  # null H
    bad = list(ptrs); bad[3] = 0x10008
    assert call_forward(p, bad) == 3                  # misaligned Wup
    assert call_forward(p, ws=0) == 8                 # no workspace
    assert call_forward(p, ws_bytes=1024) == 8        # too small
    assert call_forward(p, ws=0x100010) == 3          # workspace not 256-aligned
    assert call_forward(p, n_doc=-1) == 1
    assert call_forward(p, n_doc=3, doc=None) == 1    # doc_starts missing


def test_fp32_path_accepts_any_shape():
    L = ip.lib()
    p = params(dtype=ip.F32, d=67, F=131, C=7, T=50)
    assert L.ipttt_workspace_size(ctypes.byref(p)) > 0


def test_forward_host_size_and_argument_errors():
    L = ip.lib()
    p = params(B=2, T=777)
    size = L.ipttt_forward_host_size(ctypes.byref(p), 256, 3)
    assert size > 0 and size % 256 == 0
    assert L.ipttt_forward_host_size(ctypes.byref(p), 100, 3) == 0           # piece not a multiple of C
    assert L.ipttt_forward_host_size(ctypes.byref(params(C=96)), 0, 0) == 0  # unsupported shape
    fake = [0x10000 + 256 * i for i in range(5)]
    host = ctypes.create_string_buffer(16)
    buf = 0x100000
    # null host buffers, a bad piece length, an unsupported shape, a short device buffer
    assert L.ipttt_forward_host(ctypes.byref(p), None, None, *fake, None, 0, None, buf, size, 256, None) == 1
    assert L.ipttt_forward_host(ctypes.byref(p), host, host, *fake, None, 0, host, buf, size, 100, None) == 1
    assert L.ipttt_forward_host(ctypes.byref(params(C=96)), host, host, *fake, None, 0, host, buf, size, 0,
                                None) == 5
    assert L.ipttt_forward_host(ctypes.byref(p), host, host, *fake, None, 0, host, buf, size - 256, 256,
                                None) == 8
    # document starts are checked on the host: out of order
    docs = (ctypes.c_int32 * 2)(300, 200)
    assert L.ipttt_forward_host(ctypes.byref(p), host, host, *fake, docs, 2, host, buf, size, 256, None) == 1


def test_decode_sizes_and_argument_errors():
    L = ip.lib()
    p = params(B=4, T=1, C=128)
    assert L.ipttt_decode_state_size(ctypes.byref(p)) > 0
    assert L.ipttt_decode_host_size(ctypes.byref(p)) >= 4 * 128 * 4
    # more than 16 rows, or fp32: not supported by the decode kernels
    assert L.ipttt_decode_state_size(ctypes.byref(params(B=17))) == 0
    assert L.ipttt_decode_state_size(ctypes.byref(params(dtype=ip.F32))) == 0
    host = ctypes.create_string_buffer(L.ipttt_decode_host_size(ctypes.byref(p)))
    assert L.ipttt_decode_reset(ctypes.byref(params(B=17)), 0x100000, host, None) == 5
    assert L.ipttt_decode_reset(ctypes.byref(p), None, host, None) == 1
    assert L.ipttt_decode_reset(ctypes.byref(p), 0x100010, host, None) == 3  # misaligned state
    fake = [0x10000 + 256 * i for i in range(8)]
    # h missing
    assert L.ipttt_decode_step(ctypes.byref(p), 0x100000, host, None, fake[0], None, *fake[1:6], fake[6], None) == 1
