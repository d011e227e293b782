"""Row-sharded decode of one LiftQuant layer over a process group.

o = diag(s) . W_q . u splits by output rows (LiftQuant paper note, "Key designs" 4:
the 1-bit x float matmul has independent rows). Rank g of G keeps rows [r0_g, r1_g)
of the packed signs and of s. It runs the lift (replicated: every rank needs the
whole u) and the GEMV on its rows, and an all-gather over the group assembles o.
Shards are padded to a common height so that every rank contributes a tensor of the
same shape; padded rows have s = 0 (their output is 0) and are dropped after the
gather. The arithmetic is the library's kernels; this module only partitions rows
and assembles the gathered pieces.
"""

from __future__ import annotations


def row_range(out: int, world: int, rank: int):
    """Rows [r0, r1) of `rank`: contiguous, in rank order, sizes differing by at most one."""
    if not (world >= 1 and 0 <= rank < world and out >= world):
        raise ValueError("need out >= world >= 1 and 0 <= rank < world")
    return out * rank // world, out * (rank + 1) // world


def shard_height(out: int, world: int) -> int:
    """Common (padded) shard height: the largest shard."""
    return -(-out // world)


def assemble(pieces, out: int, world: int):
    """pieces: `world` tensors [batch][h] in rank order -> o [batch][out]; the first
    r1_g - r0_g columns of piece g are rows r0_g .. r1_g - 1 of o."""
    import torch
    cols = []
    for g, piece in enumerate(pieces):
        r0, r1 = row_range(out, world, g)
        cols.append(piece[:, : r1 - r0])
    return torch.cat(cols, dim=1)


class ShardedDecode:
    """One layer's decode step over a process group (NCCL for CUDA tensors).

    packed [out][K/32] (int32 storage of uint32) and s [out] may live on the host or
    the device; this rank copies its rows to the current device. M [d][D] and the
    whitening inverse tinv (or None) are replicated. The GEMV workspace is
    allocated once. Given `batch`, the lifted activations, the local output, the
    gather buffer and the assembled output are allocated here too, and step()
    launches no allocation (it can be captured in a CUDA graph)."""

    def __init__(self, packed, s, M, K, tinv=None, group=None, batch=None):
        import torch
        import torch.distributed as dist
        from . import gemv_workspace
        self.group = group
        self.dist = dist.is_initialized()
        self.world = dist.get_world_size(group) if self.dist else 1
        self.rank = dist.get_rank(group) if self.dist else 0
        out = int(packed.shape[0])
        r0, r1 = row_range(out, self.world, self.rank)
        h = shard_height(out, self.world)
        dev = torch.device("cuda", torch.cuda.current_device())
        self.out, self.K, self.h, self.dev = out, K, h, dev
        self.packed = torch.zeros((h, K // 32), dtype=torch.int32, device=dev)
        self.packed[: r1 - r0].copy_(packed[r0:r1])
        self.s = torch.zeros(h, dtype=torch.float32, device=dev)
        self.s[: r1 - r0].copy_(s[r0:r1])
        self.M = M.to(dev).contiguous()
        self.tinv = None if tinv is None else tinv.to(dev).contiguous()
        self._ws = {}
        self.batch = batch
        if batch is not None:
            self.u = torch.empty((batch, K), dtype=torch.float32, device=dev)
            self.o_local = torch.empty((batch, h), dtype=torch.float32, device=dev)
            self.gathered = (torch.empty((self.world, batch, h), dtype=torch.float32, device=dev)
                             if self.dist else None)
            self._workspace(batch)

    def _workspace(self, batch):
        from . import gemv_workspace
        if batch not in self._ws:
            self._ws[batch] = gemv_workspace(self.h, self.K, batch, self.dev)
        return self._ws[batch]

    def step(self, a):
        """a [batch][in] on this rank's device (batch as given at construction):
        lift, GEMV on this rank's rows, all-gather of the shard outputs into
        self.gathered [world][batch][h] (with no process group the local output
        is the whole of o); assembled() gives o."""
        import torch.distributed as dist
        from . import lift_gemv
        lift_gemv(a, self.M, self.packed, self.s, self.K, tinv=self.tinv, u=self.u, out=self.o_local,
                  workspace=self._ws[self.batch])
        if self.dist:
            dist.all_gather_into_tensor(self.gathered, self.o_local, group=self.group)

    def gemv_only(self):
        """The GEMV on this rank's rows from the lifted activations of the last step."""
        from . import gemv
        gemv(self.packed, self.s, self.u, out=self.o_local, workspace=self._ws[self.batch])

    def assembled(self):
        """o [batch][out] from the last step's gathered shard outputs."""
        if not self.dist:
            return self.o_local[:, : self.out]
        return assemble(list(self.gathered.unbind(0)), self.out, self.world)

    def __call__(self, a):
        """a [batch][in] on this rank's device -> o [batch][out] (every rank gets all of o)."""
        import torch
        import torch.distributed as dist
        from . import lift_gemv
        _, o_local = lift_gemv(a, self.M, self.packed, self.s, self.K, tinv=self.tinv,
                               workspace=self._workspace(int(a.shape[0])))
        if not self.dist:
            return o_local[:, : self.out]
        pieces = [torch.empty_like(o_local) for _ in range(self.world)]
        dist.all_gather(pieces, o_local, group=self.group)
        return assemble(pieces, self.out, self.world)
