"""B200 (sm_100a) ONNX ConvTranspose: a C-ABI CUDA library (libct.so, declared
in include/ct.h) and its thin Python binding.  ``build.build()`` compiles the
library in-tree; ``workloads`` holds the seeded synthetic inputs."""

from .ct import (  # noqa: F401
    ConvTranspose,
    CtError,
    conv_transpose,
    conv_transpose_nhwc,
    ct_output_shape,
    ct_plan,
    ct_plan_destroy,
    ct_plan_kernel,
    ct_plan_launches,
    ct_prepack_weights,
    ct_prepacked_weight_bytes,
    ct_run,
    ct_run_noalloc,
    ct_status_string,
    ct_workspace_bytes,
    make_desc,
)
