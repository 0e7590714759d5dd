"""Batch sharding of one ConvTranspose call over several GPUs.

Images are independent under ConvTranspose: Y[n] depends on X[n] alone.  A
caller's batch of N images is therefore split into contiguous slices, one
per GPU, with the weight replicated: every GPU gets its own plan and its own
pre-packed copy of W, runs the library's kernels on its own slice only, and
no data moves between GPUs during the computation.  Only a caller that needs
all of Y on one device adds one gather at the end.

Two forms:
  * ``ShardedConvTranspose``: one process per GPU (``torch.distributed``;
    NCCL on GPUs).  Rank r holds images ``shard_bounds(N, world)[r]``;
    ``gather`` assembles Y on one rank (or all) with a single all-gather of
    equal-size padded slices.
  * ``MultiDeviceConvTranspose``: one process driving a list of devices.  The
    slices are copied to their devices, each device runs its slice on its own
    current stream, and ``gather`` copies the Y slices to one device.

Every kernel only ever sees buffers of its own device: a slice of X is
copied to the device before the call, never read from a peer.
"""

import torch

from . import ct


def shard_bounds(n, world):
    """Contiguous, balanced slices of a batch of `n` images over `world`
    shards: [(lo, hi), ...], the first n % world shards one image longer."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if n < 0:
        raise ValueError("batch must be >= 0")
    base, extra = divmod(n, world)
    out, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def _shard_shape(x_shape, count):
    return [count] + list(x_shape[1:])


class ShardedConvTranspose:
    """This rank's part of a batch-sharded ConvTranspose.

    ``x_shape`` is the GLOBAL input shape (batch first in both layouts); this
    rank plans for its slice of the batch.  ``compute`` replaces the library
    call (a function of the local X slice returning the local Y slice): the
    tests use it to run the split and gather logic on the CPU.
    """

    def __init__(self, w, x_shape, bias=None, *, rank, world, device=None, compute=None,
                 process_group=None, **attrs):
        self.rank, self.world = int(rank), int(world)
        self.x_shape = list(x_shape)
        self.bounds = shard_bounds(self.x_shape[0], self.world)
        self.lo, self.hi = self.bounds[self.rank]
        self.local_shape = _shard_shape(self.x_shape, self.hi - self.lo)
        self.pg = process_group
        self._compute = compute
        self.op = None
        if compute is None and self.hi > self.lo:
            dev = torch.device(device) if device is not None else w.device
            self.op = ct.ConvTranspose(w.to(dev), self.local_shape,
                                       bias.to(dev) if bias is not None else None, **attrs)
            self.y_local_shape = list(self.op.y_shape)
        else:
            self.y_local_shape = None

    def local_slice(self, x_global):
        """This rank's images of a global batch (a view, no copy)."""
        return x_global[self.lo:self.hi]

    def __call__(self, x_local, out=None, stream=None):
        if list(x_local.shape) != self.local_shape:
            raise ValueError("X slice has shape %s, this rank holds %s"
                             % (list(x_local.shape), self.local_shape))
        if self._compute is not None:
            y = self._compute(x_local)
            self.y_local_shape = list(y.shape)
            return y
        if self.op is None:   # an empty slice (more ranks than images)
            raise ValueError("this rank holds no images; gather with y_local=None")
        return self.op(x_local, out=out, stream=stream)

    def gather(self, y_local, dst=0, all_ranks=False):
        """Assemble the global Y: one all-gather of equal-size slices (each
        rank's slice padded to the longest), then the padding dropped.
        Returns Y on rank `dst` (every rank when `all_ranks`), else None.
        Every rank must call it (a collective)."""
        import torch.distributed as dist
        longest = max(hi - lo for lo, hi in self.bounds)
        if y_local is None:
            raise ValueError("y_local is required (a rank with no images passes an empty slice)")
        tail = list(y_local.shape[1:])
        padded = y_local.new_zeros([longest] + tail)
        padded[: y_local.shape[0]] = y_local
        parts = [torch.empty_like(padded) for _ in range(self.world)]
        dist.all_gather(parts, padded.contiguous(), group=self.pg)
        if not all_ranks and self.rank != dst:
            return None
        return torch.cat([parts[r][: hi - lo] for r, (lo, hi) in enumerate(self.bounds)], dim=0)


class MultiDeviceConvTranspose:
    """One process, one plan and one packed weight per device in `devices`;
    a call splits the batch over them (see shard_bounds)."""

    def __init__(self, w, x_shape, bias=None, *, devices, **attrs):
        self.devices = [torch.device(d) for d in devices]
        self.x_shape = list(x_shape)
        self.bounds = shard_bounds(self.x_shape[0], len(self.devices))
        self.ops = []
        for (lo, hi), dev in zip(self.bounds, self.devices):
            if hi == lo:
                self.ops.append(None)
                continue
            with torch.cuda.device(dev):
                self.ops.append(ct.ConvTranspose(w.to(dev), _shard_shape(self.x_shape, hi - lo),
                                                 bias.to(dev) if bias is not None else None,
                                                 **attrs))

    def __call__(self, x):
        """Run every slice on its device (asynchronously on each device's
        current stream); returns the list of Y slices, one per device."""
        if list(x.shape) != self.x_shape:
            raise ValueError("X has shape %s, the plan was made for %s" % (list(x.shape), self.x_shape))
        ys = []
        for (lo, hi), dev, op in zip(self.bounds, self.devices, self.ops):
            if op is None:
                ys.append(None)
                continue
            with torch.cuda.device(dev):
                xs = x[lo:hi].to(dev, non_blocking=True)
                ys.append(op(xs))
        return ys

    def gather(self, ys, device=None):
        """Concatenate the Y slices on one device (the first by default)."""
        dev = torch.device(device) if device is not None else self.devices[0]
        return torch.cat([y.to(dev, non_blocking=True) for y in ys if y is not None], dim=0)
