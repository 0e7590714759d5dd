"""Random small ConvTranspose cases for sweeps (test-side only)."""

import numpy as np

from oracle import Attrs, ResolveError, resolve_full


def attrs_of(case):
    return Attrs(strides=case["strides"], dilations=case.get("dilations"),
                 pads=case.get("pads"), output_padding=case.get("output_padding"),
                 auto_pad=case.get("auto_pad", "NOTSET"), group=case.get("group", 1),
                 kernel_shape=case.get("kernel_shape"),
                 output_shape=case.get("output_shape"))


def random_case(rng, max_rank=3, max_cg=3, max_mg=3, lim_in=None, lim_k=None,
                groups=(1, 1, 2, 4), strides=(1, 5), dils=(1, 4), pads=(-1, 3)):
    """One random attribute set whose output is non-empty (rejection sampled)."""
    while True:
        rank = int(rng.integers(1, max_rank + 1))
        g = int(rng.choice(list(groups)))
        cg = int(rng.integers(1, max_cg + 1))
        mg = int(rng.integers(1, max_mg + 1))
        n = int(rng.integers(1, 3))
        li = (lim_in or {1: 12, 2: 7, 3: 4})[rank]
        lk = (lim_k or {1: 5, 2: 4, 3: 3})[rank]
        ins = [int(rng.integers(1, li + 1)) for _ in range(rank)]
        ks = [int(rng.integers(1, lk + 1)) for _ in range(rank)]
        ss = [int(rng.integers(*strides)) for _ in range(rank)]
        ds = [int(rng.integers(*dils)) for _ in range(rank)]
        ops = [int(rng.integers(0, max(ss[a], ds[a]))) for a in range(rank)]
        pp = [int(rng.integers(*pads)) for _ in range(2 * rank)]
        case = dict(x_shape=[n, cg * g] + ins, w_shape=[cg * g, mg] + ks,
                    strides=ss, dilations=ds, pads=pp, output_padding=ops,
                    group=g, bias=bool(rng.integers(0, 2)))
        try:
            resolve_full(case["x_shape"], case["w_shape"], attrs_of(case))
        except ResolveError:
            continue
        return case
