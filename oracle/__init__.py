"""Independent fp64 CPU oracle for ONNX ConvTranspose.

TEST INFRASTRUCTURE ONLY: ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may use it; the CUDA library and its Python
binding never import it.  It shares no code, tables or helpers with the CUDA
path.

Every function is pinned by CPU tests to something other than itself:
hand-worked examples under tests/golden/, the shape rules of the
ai.onnx.ConvTranspose README, the stride-1 and adjoint identities, 1x1 =
matmul, and PyTorch's CPU conv_transpose in fp64 as a library special case
(with torch.relu for the ReLU activation).
"""

from .resolver import Attrs, Resolved, ResolveError, resolve, resolve_full  # noqa: F401
from .reference import (  # noqa: F401
    ACTIVATIONS,
    apply_activation,
    build,
    conv_transpose_points,
    conv_transpose_ref,
    forward_conv_ref,
    to_channels_first,
)
