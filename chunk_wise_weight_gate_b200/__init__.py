"""In-Place Test-Time Training MLP layer forward for NVIDIA B200 (sm_100a).

The layer: a gated MLP whose down projection is a fast weight, updated chunk by
chunk with a clipped Hebbian delta from an LM-aligned target and reset at each
document start.  All arithmetic runs in libipttt.so (hand-written CUDA); this
package only marshals arguments (ipttt.py) and draws seeded synthetic inputs
(synth.py).
"""
from .ipttt import (BF16, F32, IptttError, LayerConfig, StreamState, alloc_workspace, core, flops_per_token,
                    forward, get_status, lib, version, workspace_size)

__all__ = ["BF16", "F32", "IptttError", "LayerConfig", "StreamState", "alloc_workspace", "core",
           "flops_per_token", "forward", "get_status", "lib", "version", "workspace_size"]
