"""Tensor-parallel sharding of the W4A16 product over P devices.

Page 4 (llm-glossary.tokens-kit.com, quantization methods, the production
checklist) asks that tensor-parallel shards agree with the quantization groups
and with which device owns each scale.  A linear layer Y = X . W^T with
W [N, K] is split in one of two ways:

  column-parallel ("n"): device r owns rows [n0, n1) of W (its own qweight,
      scales and zero-point rows), reads all of X and computes Y[:, n0:n1].
      Groups run along k, so every row split keeps every group whole.  An
      all-gather gives each device the whole Y when the consumer needs it.
  row-parallel ("k"): device r owns columns [k0, k1) of W and of X.  K / P must
      be a multiple of the group size g, so that each group -- and its scale
      and zero-point -- lives on exactly one device; a split that would cut a
      group is rejected on the host (ShardError) before anything runs.  Each
      device computes the fp32 partial X[:, k0:k1] . W^[:, k0:k1]^T
      (W4_OUT_F32), an all-reduce adds the partials, and the sum is rounded to
      bf16 once (w4_f32_to_bf16).

A shard is quantized from its own slice of W; by the group alignment above
this gives the same codes, scales and zero-points as slicing the quantization
of the whole matrix.  The collectives are torch.distributed calls (NCCL over
NVLink on B200s); no kernel reads a peer's memory and nothing uses multicast.
The local quantization and product default to this library's kernels; a
caller may pass another implementation with the same four methods (`ops`),
which is how the multi-process tests run the plumbing on CPU processes.
"""
from __future__ import annotations

SPLITS = ("n", "k")


class ShardError(ValueError):
    """A split that the shards cannot own consistently."""


def n_range(N: int, P: int, rank: int) -> tuple[int, int]:
    """Rows [n0, n1) of device `rank`: P contiguous ranges, the first N % P one
    row longer."""
    if P < 1 or not 0 <= rank < P:
        raise ShardError("rank %d outside 0..%d" % (rank, P - 1))
    if N < P:
        raise ShardError("N = %d rows cannot be split over %d devices" % (N, P))
    base, extra = divmod(N, P)
    n0 = rank * base + min(rank, extra)
    return n0, n0 + base + (1 if rank < extra else 0)


def k_range(K: int, P: int, rank: int, group: int) -> tuple[int, int]:
    """Columns [k0, k1) of device `rank` for a row-parallel split: K / P must be
    a whole number of groups of `group` columns."""
    if P < 1 or not 0 <= rank < P:
        raise ShardError("rank %d outside 0..%d" % (rank, P - 1))
    if K % P != 0 or (K // P) % group != 0:
        raise ShardError("K = %d over %d devices gives %s columns per device, not a multiple of the group size %d: "
                         "a group and its scale would straddle two devices" % (K, P, K / P, group))
    w = K // P
    return rank * w, (rank + 1) * w


class LibraryOps:
    """The local steps on this library's kernels (CUDA tensors)."""

    def __init__(self):
        import bit_gemm_quant_b200 as w4
        self.w4 = w4

    def quant_pack(self, W, group, mode, s=None):
        return self.w4.quant_pack(W, group, mode, s=s)

    def gemm(self, X, packed, group, mode, N, out_f32=False):
        q, sc, z = packed
        return self.w4.gemm(X, q, sc, z, group, mode, N=N, out_f32=out_f32)

    def f32_to_bf16(self, Y):
        return self.w4.f32_to_bf16(Y)

    def empty(self, shape, like, dtype):
        import torch
        return torch.empty(shape, dtype=dtype, device=like.device)


class ShardedW4Linear:
    """One device's share of a quantized linear layer.

    W_local is this device's slice of the bf16 weight: rows [n0, n1) for split
    "n", columns [k0, k1) for split "k" (see local_weight).  forward() takes
    this device's activations (all of X for "n", X[:, k0:k1] for "k") and
    returns the whole bf16 Y on every device (gather=True), or only this
    device's columns of Y (split "n", gather=False)."""

    def __init__(self, W_local, N: int, K: int, group: int, mode: int, split: str, P: int, rank: int,
                 s_local=None, process_group=None, ops=None):
        if split not in SPLITS:
            raise ShardError("split must be one of %s" % (SPLITS,))
        self.N, self.K, self.group, self.mode, self.split, self.P, self.rank = N, K, group, mode, split, P, rank
        self.pg = process_group
        self.ops = ops if ops is not None else LibraryOps()
        if split == "n":
            self.n0, self.n1 = n_range(N, P, rank)
            self.k0, self.k1 = 0, K
        else:
            self.n0, self.n1 = 0, N
            self.k0, self.k1 = k_range(K, P, rank, group)
        want = (self.n1 - self.n0, self.k1 - self.k0)
        if tuple(W_local.shape) != want:
            raise ShardError("local weight has shape %s, this shard is %s" % (tuple(W_local.shape), want))
        self.packed = self.ops.quant_pack(W_local, group, mode, s_local)

    def forward(self, X_local, gather: bool = True):
        import torch
        import torch.distributed as dist
        if self.split == "n":
            Y = self.ops.gemm(X_local, self.packed, self.group, self.mode, self.n1 - self.n0)
            if not gather or self.P == 1:
                return Y
            # equal-sized pieces for the all-gather: pad to the longest shard
            M = Y.shape[0]
            width = n_range(self.N, self.P, 0)[1]
            piece = Y if Y.shape[1] == width else torch.nn.functional.pad(Y, (0, width - Y.shape[1]))
            # gathered as bytes: a bit copy whatever the backend's bf16 support
            esz = piece.element_size()
            raw = piece.contiguous().view(torch.uint8)
            parts = [self.ops.empty((M, width * esz), raw, torch.uint8) for _ in range(self.P)]
            dist.all_gather(parts, raw, group=self.pg)
            cols = []
            for r, p in enumerate(parts):
                a, b = n_range(self.N, self.P, r)
                cols.append(p[:, :(b - a) * esz])
            return torch.cat(cols, dim=1).view(Y.dtype)
        partial = self.ops.gemm(X_local, self.packed, self.group, self.mode, self.N, out_f32=True)
        if self.P > 1:
            dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=self.pg)
        return self.ops.f32_to_bf16(partial)


def _contig(a):
    return a.contiguous() if hasattr(a, "contiguous") else a.copy()


def local_weight(W, split: str, P: int, rank: int, group: int):
    """This device's slice of the full weight W [N, K] (a view for "n", a
    contiguous copy for "k")."""
    N, K = W.shape
    if split == "n":
        n0, n1 = n_range(N, P, rank)
        return W[n0:n1]
    k0, k1 = k_range(K, P, rank, group)
    return _contig(W[:, k0:k1])


def local_activations(X, split: str, P: int, rank: int, group: int):
    """This device's activations: all of X for "n", X[:, k0:k1] for "k"."""
    if split == "n":
        return X
    k0, k1 = k_range(X.shape[1], P, rank, group)
    return _contig(X[:, k0:k1])


def local_smoothing(s, split: str, P: int, rank: int, group: int):
    """This device's part of a smoothing vector s [K] (folded along k)."""
    if s is None or split == "n":
        return s
    k0, k1 = k_range(s.shape[0], P, rank, group)
    return _contig(s[k0:k1])
