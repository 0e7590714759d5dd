"""Python binding of libct.so (include/ct.h): argument marshalling only.

The functions carry the C names (``ct_output_shape``, ``ct_plan``,
``ct_prepack_weights``, ``ct_run`` ...) and take plain integers for device
pointers and streams.  ``ConvTranspose`` wraps them for torch tensors: torch
provides the device memory and the stream, every step of the operator runs
in the library's CUDA kernels.  There is no fallback: when libct.so is
missing or the device is not an sm_100 part, calls raise.

Attribute names follow the ai.onnx.ConvTranspose README ("Attributes");
``conv_transpose_nhwc`` follows ClikaRT::ops::conv_transpose (channels-last,
weight [C_in, K.., O/groups], padding as (lo, hi) per spatial dim).
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libct.so")

CT_OK = 0
STATUS_NAMES = {0: "CT_OK", 1: "CT_ERR_CHANNELS", 2: "CT_ERR_SPAN", 3: "CT_ERR_DTYPE",
                4: "CT_ERR_ATTR", 5: "CT_ERR_ALIGN", 6: "CT_ERR_NULL", 7: "CT_ERR_DEVICE",
                8: "CT_ERR_WORKSPACE", 9: "CT_ERR_UNSUPPORTED", 10: "CT_ERR_NOMEM"}
CT_F32, CT_F16 = 0, 1
CT_NCHW, CT_NHWC = 0, 1
AUTOPAD = {"NOTSET": 0, "SAME_UPPER": 1, "SAME_LOWER": 2, "VALID": 3}
ALGO = {"auto": 0, "generic": 1, "dense_tc": 2, "fp32_gemm": 3, "grouped": 4,
        "dense_tc_pertap": 5, "dense_tc_pair": 6}

PART_PREPARE, PART_MAIN, PART_ALL = 1, 2, 3

EXPORTED = ["ct_output_shape", "ct_plan", "ct_plan_kernel", "ct_plan_launches",
            "ct_prepacked_weight_bytes",
            "ct_workspace_bytes", "ct_prepack_weights", "ct_run", "ct_run_parts",
            "ct_run_noalloc", "ct_plan_destroy", "ct_status_string", "ct_take_device_error",
            "ct_selftest_wait_timeout"]


class CtError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (%s)" % (where, STATUS_NAMES.get(status, status),
                                          ct_status_string(status)))


class ct_desc(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("layout", ctypes.c_int32), ("auto_pad", ctypes.c_int32),
                ("N", ctypes.c_int64), ("C", ctypes.c_int64),
                ("in_", ctypes.c_int64 * 3), ("w_dims", ctypes.c_int64 * 5),
                ("group", ctypes.c_int64), ("bias_len", ctypes.c_int64),
                ("strides", ctypes.c_int64 * 3), ("dilations", ctypes.c_int64 * 3),
                ("pads", ctypes.c_int64 * 6), ("output_padding", ctypes.c_int64 * 3),
                ("has_kernel_shape", ctypes.c_int32), ("has_output_shape", ctypes.c_int32),
                ("kernel_shape", ctypes.c_int64 * 3), ("output_shape", ctypes.c_int64 * 3),
                ("algo", ctypes.c_int32), ("activation", ctypes.c_int32)]


_lib = None


def lib():
    """Load libct.so (raises when it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libct.so is not built (%s); run "
                              "transposed_convolution_02_b200/build.py" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        i64p = ctypes.POINTER(ctypes.c_int64)
        szp = ctypes.POINTER(ctypes.c_size_t)
        dp = ctypes.POINTER(ct_desc)
        L.ct_output_shape.argtypes = [dp, i64p, i64p, i64p]
        L.ct_plan.argtypes = [dp, ctypes.POINTER(P)]
        L.ct_plan_kernel.argtypes = [P]
        L.ct_plan_kernel.restype = ctypes.c_char_p
        L.ct_plan_launches.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
        L.ct_prepacked_weight_bytes.argtypes = [P, szp]
        L.ct_workspace_bytes.argtypes = [P, szp]
        L.ct_prepack_weights.argtypes = [P, P, P, P]
        L.ct_run.argtypes = [P, P, P, P, P, P, P]
        L.ct_run_parts.argtypes = [P, P, P, P, P, P, P, ctypes.c_int32]
        L.ct_selftest_wait_timeout.argtypes = [P, ctypes.c_int64]
        L.ct_run_noalloc.argtypes = [P, P, P, P, P, P]
        L.ct_plan_destroy.argtypes = [P]
        L.ct_plan_destroy.restype = None
        L.ct_take_device_error.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
        L.ct_status_string.argtypes = [ctypes.c_int]
        L.ct_status_string.restype = ctypes.c_char_p
        for name in ("ct_output_shape", "ct_plan", "ct_plan_launches", "ct_prepacked_weight_bytes",
                     "ct_workspace_bytes", "ct_prepack_weights", "ct_run", "ct_run_parts",
                     "ct_run_noalloc", "ct_take_device_error", "ct_selftest_wait_timeout"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


# ---- the C entry points, same names -------------------------------------

def ct_status_string(status):
    return lib().ct_status_string(int(status)).decode()


def ct_output_shape(desc):
    y = (ctypes.c_int64 * 5)()
    pb = (ctypes.c_int64 * 3)()
    pe = (ctypes.c_int64 * 3)()
    st = lib().ct_output_shape(ctypes.byref(desc), y, pb, pe)
    if st != CT_OK:
        raise CtError(st, "ct_output_shape")
    r = desc.rank
    return list(y)[: r + 2], list(pb)[:r], list(pe)[:r]


def ct_plan(desc):
    h = ctypes.c_void_p()
    st = lib().ct_plan(ctypes.byref(desc), ctypes.byref(h))
    if st != CT_OK:
        raise CtError(st, "ct_plan")
    return h


def ct_plan_kernel(plan):
    return lib().ct_plan_kernel(plan).decode()


def ct_plan_launches(plan):
    n = ctypes.c_int32()
    st = lib().ct_plan_launches(plan, ctypes.byref(n))
    if st != CT_OK:
        raise CtError(st, "ct_plan_launches")
    return n.value


def ct_prepacked_weight_bytes(plan):
    n = ctypes.c_size_t()
    st = lib().ct_prepacked_weight_bytes(plan, ctypes.byref(n))
    if st != CT_OK:
        raise CtError(st, "ct_prepacked_weight_bytes")
    return n.value


def ct_workspace_bytes(plan):
    n = ctypes.c_size_t()
    st = lib().ct_workspace_bytes(plan, ctypes.byref(n))
    if st != CT_OK:
        raise CtError(st, "ct_workspace_bytes")
    return n.value


def ct_prepack_weights(plan, w_ptr, wp_ptr, stream):
    st = lib().ct_prepack_weights(plan, w_ptr, wp_ptr, stream)
    if st != CT_OK:
        raise CtError(st, "ct_prepack_weights")


def ct_run(plan, x_ptr, wp_ptr, bias_ptr, y_ptr, ws_ptr, stream):
    st = lib().ct_run(plan, x_ptr, wp_ptr, bias_ptr, y_ptr, ws_ptr, stream)
    if st != CT_OK:
        raise CtError(st, "ct_run")


def ct_run_parts(plan, x_ptr, wp_ptr, bias_ptr, y_ptr, ws_ptr, stream, parts):
    """ct_run restricted to a mask of PART_PREPARE (re-layout, bias fill) and
    PART_MAIN (the main kernel), for timing the parts of a call apart."""
    st = lib().ct_run_parts(plan, x_ptr, wp_ptr, bias_ptr, y_ptr, ws_ptr, stream, int(parts))
    if st != CT_OK:
        raise CtError(st, "ct_run_parts")


def ct_selftest_wait_timeout(limit_cycles, stream=None):
    """Launch the bounded-wait self-test (a wait that gives up after
    `limit_cycles` SM cycles, then drains its copy in flight); the next
    ct_take_device_error() returns 501."""
    st = lib().ct_selftest_wait_timeout(_stream_ptr(stream), int(limit_cycles))
    if st != CT_OK:
        raise CtError(st, "ct_selftest_wait_timeout")


def ct_run_noalloc(plan, x_ptr, wp_ptr, bias_ptr, y_ptr, stream):
    """ct_run with the workspace taken from the library's fixed device array
    (for callers that may not allocate device memory while running)."""
    st = lib().ct_run_noalloc(plan, x_ptr, wp_ptr, bias_ptr, y_ptr, stream)
    if st != CT_OK:
        raise CtError(st, "ct_run_noalloc")


def ct_take_device_error(stream=None):
    """Wait for the stream, then read and clear the kernels' device error
    words: 0 when no bounded wait ran out since the last call, else the code
    100 * module + wait site.  Raises CtError when a CUDA call failed."""
    code = ctypes.c_int32()
    st = lib().ct_take_device_error(_stream_ptr(stream) if torch.cuda.is_available() else None,
                                    ctypes.byref(code))
    if st != CT_OK and code.value == 0:
        raise CtError(st, "ct_take_device_error")
    return code.value


def ct_plan_destroy(plan):
    if plan:
        lib().ct_plan_destroy(plan)


# ---- descriptor construction ----------------------------------------------

ACTIVATION = {"identity": 0, "relu": 1}


def make_desc(x_shape, w_shape, *, dtype, layout="nchw", strides=None, dilations=None,
              pads=None, output_padding=None, auto_pad="NOTSET", group=1, bias_len=0,
              kernel_shape=None, output_shape=None, algo="auto", activation="identity"):
    """Fill a ct_desc from tensor shapes and README-named attributes."""
    d = ct_desc()
    r = len(x_shape) - 2
    d.rank = r
    d.dtype = {torch.float32: CT_F32, torch.float16: CT_F16}.get(dtype, 99)
    d.layout = CT_NCHW if layout == "nchw" else CT_NHWC
    d.auto_pad = AUTOPAD.get(auto_pad, 99)
    d.N = int(x_shape[0])
    if layout == "nchw":
        d.C = int(x_shape[1])
        sp = x_shape[2:]
    else:
        d.C = int(x_shape[-1])
        sp = x_shape[1:-1]
    for a in range(min(r, 3)):
        d.in_[a] = int(sp[a])
    for a, v in enumerate(list(w_shape)[:5]):
        d.w_dims[a] = int(v)
    d.group = int(group)
    d.bias_len = int(bias_len)
    for a in range(min(r, 3)):
        d.strides[a] = int(strides[a]) if strides is not None else 1
        d.dilations[a] = int(dilations[a]) if dilations is not None else 1
        d.output_padding[a] = int(output_padding[a]) if output_padding is not None else 0
    if pads is not None:
        for a, v in enumerate(list(pads)[:6]):
            d.pads[a] = int(v)
    if kernel_shape is not None:
        d.has_kernel_shape = 1
        for a, v in enumerate(list(kernel_shape)[:3]):
            d.kernel_shape[a] = int(v)
    if output_shape is not None:
        d.has_output_shape = 1
        for a, v in enumerate(list(output_shape)[:3]):
            d.output_shape[a] = int(v)
    d.algo = ALGO[algo]
    d.activation = ACTIVATION.get(activation, 99)
    return d


# ---- torch-facing wrapper ---------------------------------------------------

def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream_ptr(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def check_io(x, out, x_shape, y_shape, dtype, device):
    """Refuse a call whose tensors do not match the plan (the kernels trust the
    planned sizes: a different X or Y would be read or written out of bounds)."""
    if list(x.shape) != list(x_shape):
        raise ValueError("X has shape %s, the plan was made for %s" % (list(x.shape), list(x_shape)))
    if x.dtype != dtype:
        raise ValueError("X is %s, the plan computes in %s" % (x.dtype, dtype))
    if x.device != device:
        raise ValueError("X is on %s, the packed weights on %s" % (x.device, device))
    if out is not None:
        if list(out.shape) != list(y_shape) or out.dtype != dtype or out.device != device:
            raise ValueError("out must be a %s tensor of shape %s on %s" % (dtype, list(y_shape), device))
        if not out.is_contiguous():
            raise ValueError("out must be contiguous")


class ConvTranspose:
    """A planned ConvTranspose with its weight pre-packed on the device.

    Plan and pre-pack happen once here; ``__call__`` allocates Y (and the
    workspace once) with torch and launches ``ct_run`` on the current stream.
    """

    def __init__(self, w, x_shape, bias=None, *, layout="nchw", strides=None, dilations=None,
                 pads=None, output_padding=None, auto_pad="NOTSET", group=1,
                 kernel_shape=None, output_shape=None, algo="auto", activation="identity",
                 stream=None):
        if not w.is_cuda:
            raise ValueError("W must be a CUDA tensor")
        if bias is not None and (bias.dtype != w.dtype or bias.device != w.device):
            raise ValueError("bias must be a tensor of W's dtype on W's device")
        self.layout = layout
        self.dtype = w.dtype
        self.device = w.device
        self.x_shape = list(x_shape)
        self.desc = make_desc(list(x_shape), list(w.shape), dtype=w.dtype, layout=layout,
                              strides=strides, dilations=dilations, pads=pads,
                              output_padding=output_padding, auto_pad=auto_pad, group=group,
                              bias_len=0 if bias is None else bias.numel(),
                              kernel_shape=kernel_shape, output_shape=output_shape, algo=algo,
                              activation=activation)
        self.y_shape, self.pad_begin, self.pad_end = ct_output_shape(self.desc)
        self.plan = ct_plan(self.desc)
        self.kernel = ct_plan_kernel(self.plan)
        self.launches = ct_plan_launches(self.plan)
        nb = ct_prepacked_weight_bytes(self.plan)
        self.w_packed = torch.empty(max(nb, 16), dtype=torch.uint8, device=w.device)
        ws = ct_workspace_bytes(self.plan)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=w.device) if ws else None
        self.bias = bias.contiguous() if bias is not None else None
        w = w.contiguous()
        ct_prepack_weights(self.plan, _ptr(w), _ptr(self.w_packed), _stream_ptr(stream))
        self._w_keep = w

    def __call__(self, x, out=None, stream=None):
        if not x.is_cuda:
            raise ValueError("X must be a CUDA tensor")
        check_io(x, out, self.x_shape, self.y_shape, self.dtype, self.device)
        x = x.contiguous()
        y = out if out is not None else torch.empty(self.y_shape, dtype=self.dtype,
                                                    device=x.device)
        ct_run(self.plan, _ptr(x), _ptr(self.w_packed), _ptr(self.bias), _ptr(y),
               _ptr(self.workspace), _stream_ptr(stream))
        return y

    def run_ptrs(self, x_ptr, y_ptr, stream_ptr, parts=PART_ALL):
        """Launch on raw device pointers (benchmark loops); the caller
        guarantees buffers of the planned shapes, dtype and device.  `parts`
        restricts the call to its preparation or main launches."""
        ct_run_parts(self.plan, x_ptr, _ptr(self.w_packed), _ptr(self.bias), y_ptr,
                     _ptr(self.workspace), stream_ptr, parts)

    def run_part(self, x, out, parts, stream=None):
        """ct_run_parts on tensors checked against the plan (see run_ptrs)."""
        check_io(x, out, self.x_shape, self.y_shape, self.dtype, self.device)
        if out is None or not x.is_contiguous():
            raise ValueError("run_part needs a contiguous X and an out tensor")
        ct_run_parts(self.plan, _ptr(x), _ptr(self.w_packed), _ptr(self.bias), _ptr(out),
                     _ptr(self.workspace), _stream_ptr(stream), parts)
        return out

    def __del__(self):
        try:
            ct_plan_destroy(self.plan)
        except Exception:
            pass


def conv_transpose(x, w, bias=None, *, strides=None, dilations=None, pads=None,
                   output_padding=None, auto_pad="NOTSET", group=1, kernel_shape=None,
                   output_shape=None, algo="auto", activation="identity"):
    """ONNX ConvTranspose, channels-first: X[N,C,D..], W[C,M/group,k..] -> Y
    (optionally followed by the activation, identity by default)."""
    op = ConvTranspose(w, list(x.shape), bias, layout="nchw", strides=strides,
                       dilations=dilations, pads=pads, output_padding=output_padding,
                       auto_pad=auto_pad, group=group, kernel_shape=kernel_shape,
                       output_shape=output_shape, algo=algo, activation=activation)
    return op(x)


def conv_transpose_nhwc(x, w, bias=None, *, stride, padding, output_padding, groups,
                        dilation, activation="identity", algo="auto"):
    """Channels-last call in the form of ClikaRT::ops::conv_transpose: input
    [N, D.., C_in], weight [C_in, K.., O/groups], padding (lo, hi) per spatial
    dim, activation (identity or relu), output [N, out.., C_out]."""
    r = x.dim() - 2
    if len(padding) != 2 * r:
        raise ValueError("padding needs two entries (lo, hi) per spatial dim")
    pads = [padding[2 * a] for a in range(r)] + [padding[2 * a + 1] for a in range(r)]
    op = ConvTranspose(w, list(x.shape), bias, layout="nhwc", strides=stride,
                       dilations=dilation, pads=pads, output_padding=output_padding,
                       group=groups, algo=algo, activation=activation)
    return op(x)
