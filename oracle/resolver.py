"""Output-size and padding resolver of the oracle (test infrastructure only).

Independent of the CUDA library's own resolver: the two share no code.

Sources (ai.onnx.ConvTranspose README, "Attributes" table):
  * ``pads``: begins of every spatial axis, then ends; default zeros.
  * ``output_padding``: extra size on the high end of each axis, each value
    smaller than the stride or the dilation of that axis.
  * ``auto_pad``: NOTSET uses ``pads``; SAME_UPPER / SAME_LOWER make the
    output size equal input size times stride, the odd extra unit of padding
    going to the end (UPPER) or the beginning (LOWER); VALID pads nothing.
  * ``kernel_shape``: optional, must equal W's spatial dims.
  * ``output_shape``: optional requested output spatial dims.
The pages print no size formula.  The one used here, per axis,

    out = stride * (in - 1) + output_padding + (k - 1) * dilation + 1
          - pad_begin - pad_end

is what the scatter definition gives: the last input (in - 1) with the last
tap (k - 1) lands at stride*(in-1) - pad_begin + (k-1)*dilation, the output
covers that position, and ``output_padding`` adds to the high end.

Readings where the pages are silent (each also listed in the design notes):
  * a SAME split puts the odd unit of the total (with its sign) at the stated
    end: half = total truncated toward zero / 2;
  * ``output_shape`` derives the pads from total = natural size - requested
    size, split like SAME_LOWER when auto_pad is SAME_LOWER and otherwise with
    the odd unit at the end; explicit pads are then ignored;
  * explicit non-zero pads together with auto_pad != NOTSET are rejected;
  * VALID with an ``output_shape`` that differs from the natural size is
    rejected.
"""

from dataclasses import dataclass, field
from typing import Optional, Sequence


class ResolveError(ValueError):
    """Raised for an inconsistent attribute set."""


def _split_total(total: int, odd_at_end: bool):
    # Truncating halving so that the odd unit, with its sign, sits at the
    # requested end for negative totals too.
    half = total // 2 if total >= 0 else -((-total) // 2)
    extra = total - 2 * half
    if odd_at_end:
        return half, half + extra
    return half + extra, half


@dataclass
class Attrs:
    strides: Sequence[int]
    dilations: Optional[Sequence[int]] = None
    pads: Optional[Sequence[int]] = None          # ONNX order: begins, then ends
    output_padding: Optional[Sequence[int]] = None
    auto_pad: str = "NOTSET"
    group: int = 1
    kernel_shape: Optional[Sequence[int]] = None
    output_shape: Optional[Sequence[int]] = None


@dataclass
class Resolved:
    out: list = field(default_factory=list)
    pad_begin: list = field(default_factory=list)
    pad_end: list = field(default_factory=list)


def resolve(in_spatial, k_spatial, attrs: Attrs) -> Resolved:
    """Resolve output spatial sizes and begin/end pads for one call."""
    r = len(in_spatial)
    if len(k_spatial) != r:
        raise ResolveError("span: kernel rank differs from input rank")
    s = list(attrs.strides) if attrs.strides is not None else [1] * r
    d = list(attrs.dilations) if attrs.dilations is not None else [1] * r
    op = list(attrs.output_padding) if attrs.output_padding is not None else [0] * r
    pads = list(attrs.pads) if attrs.pads is not None else [0] * (2 * r)
    if len(s) != r or len(d) != r or len(op) != r or len(pads) != 2 * r:
        raise ResolveError("span: attribute length differs from the spatial rank")
    if attrs.kernel_shape is not None:
        if len(attrs.kernel_shape) != r:
            raise ResolveError("span: kernel_shape length")
        if list(attrs.kernel_shape) != list(k_spatial):
            raise ResolveError("attr: kernel_shape differs from W's spatial dims")
    for a in range(r):
        if s[a] <= 0 or d[a] <= 0 or k_spatial[a] <= 0 or in_spatial[a] < 0:
            raise ResolveError("attr: stride, dilation and kernel must be positive")
        if op[a] < 0 or op[a] >= max(s[a], d[a]):
            raise ResolveError("attr: output_padding must be below max(stride, dilation)")
    mode = attrs.auto_pad
    if mode not in ("NOTSET", "SAME_UPPER", "SAME_LOWER", "VALID"):
        raise ResolveError("attr: unknown auto_pad")
    if mode != "NOTSET" and any(p != 0 for p in pads):
        raise ResolveError("attr: explicit pads together with auto_pad")

    natural = [s[a] * (in_spatial[a] - 1) + op[a] + (k_spatial[a] - 1) * d[a] + 1
               for a in range(r)]
    res = Resolved()
    if attrs.output_shape is not None:
        if len(attrs.output_shape) != r:
            raise ResolveError("span: output_shape length")
        for a in range(r):
            want = attrs.output_shape[a]
            if mode == "VALID":
                if want != natural[a]:
                    raise ResolveError("attr: output_shape contradicts VALID")
                pb, pe = 0, 0
            else:
                pb, pe = _split_total(natural[a] - want, odd_at_end=(mode != "SAME_LOWER"))
            res.pad_begin.append(pb)
            res.pad_end.append(pe)
    else:
        for a in range(r):
            if mode == "NOTSET":
                pb, pe = pads[a], pads[r + a]
            elif mode == "VALID":
                pb, pe = 0, 0
            else:
                total = natural[a] - in_spatial[a] * s[a]
                pb, pe = _split_total(total, odd_at_end=(mode == "SAME_UPPER"))
            res.pad_begin.append(pb)
            res.pad_end.append(pe)
    for a in range(r):
        o = natural[a] - res.pad_begin[a] - res.pad_end[a]
        if o <= 0:
            raise ResolveError("attr: output size must be positive")
        res.out.append(o)
    return res


def resolve_full(x_shape, w_shape, attrs: Attrs, bias_len: Optional[int] = None):
    """Check channel/group arithmetic for channels-first X, W and return
    (Y shape, Resolved).  X[N, C, D..], W[C, M/group, k..], bias length M."""
    if len(x_shape) < 3 or len(x_shape) > 5 or len(w_shape) != len(x_shape):
        raise ResolveError("span: X and W must both have rank 3..5")
    n, c = x_shape[0], x_shape[1]
    g = attrs.group
    if g <= 0 or c % g != 0 or w_shape[0] != c:
        raise ResolveError("channels: C must equal W[0] and divide by group")
    m = w_shape[1] * g
    if bias_len is not None and bias_len != m:
        raise ResolveError("channels: bias length differs from M")
    res = resolve(list(x_shape[2:]), list(w_shape[2:]), attrs)
    return [n, m] + res.out, res
