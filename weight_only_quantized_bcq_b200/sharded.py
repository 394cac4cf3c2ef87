"""Tensor-parallel LUT-GEMM: one BCQ matrix split over the ranks of a process group.

The product y = sum_i alpha_i * (B_i x) splits two ways without changing what
any rank computes (LUT-GEMM card, Key points: OPT-175B generation on eight GPUs
for the FP16 baseline against one GPU for 3-bit LUT-GEMM; the matmul share of
decode time in the Fig. 5 caption):

* **Rows** (split m).  A rank holds the planes and scales of a contiguous range
  of rows, 32-row tiles at a time.  x is the same on every rank; each rank's
  output rows are gathered (all-gather).
* **Inputs** (split n).  A rank holds the planes and scales of a contiguous
  range of inputs, whole scale groups at a time, and takes the matching slice
  of x.  Its product is a partial sum of every output row; the partials are
  summed (all-reduce) or summed and split by rows (reduce-scatter).

A two-layer block pairs them (the usual tensor-parallel MLP): the first matrix
split by rows leaves each rank with a slice of the hidden vector, which is
exactly the input slice of the second matrix split by inputs, so the block
needs one all-reduce and no exchange in between.

Each rank's product is ``lutgemm.run`` on its own shard (the CUDA library);
the exchange is a ``torch.distributed`` collective on the same stream (NCCL
over NVLink on GPUs).  The shard arithmetic and the collectives are plain host
code; ``local_product`` may be replaced for testing that logic without a GPU.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

ROW_ALIGN = 32          # row tile of the packed layout


@dataclass(frozen=True)
class ShardPlan:
    """Which part of an m x n BCQ matrix (q planes, groups of g) a rank holds."""

    kind: str           # "rows" or "inputs"
    m: int
    n: int
    q: int
    g: int
    world: int
    rank: int
    lo: int             # first row (rows) or input (inputs) of this rank
    hi: int             # one past the last
    span: int           # the largest range over all ranks (gather padding)

    @property
    def local_m(self) -> int:
        return self.hi - self.lo if self.kind == "rows" else self.m

    @property
    def local_n(self) -> int:
        return self.hi - self.lo if self.kind == "inputs" else self.n


def _split(units: int, world: int, rank: int):
    """Contiguous near-equal split of `units` over `world` ranks (earlier ranks
    take the remainder): (first unit, one past the last, largest count)."""
    base, rem = divmod(units, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0), base + (1 if rem else 0)


def plan_rows(m: int, n: int, q: int, g: int, world: int, rank: int) -> ShardPlan:
    """Rows in whole 32-row tiles; the last rank's range ends at m."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    tiles = -(-m // ROW_ALIGN)
    t0, t1, tspan = _split(tiles, world, rank)
    lo, hi = min(m, t0 * ROW_ALIGN), min(m, t1 * ROW_ALIGN)
    return ShardPlan("rows", m, n, q, g, world, rank, lo, hi, tspan * ROW_ALIGN)


def plan_inputs(m: int, n: int, q: int, g: int, world: int, rank: int) -> ShardPlan:
    """Inputs in whole scale groups (each rank's n stays a multiple of g)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    if n % g:
        raise ValueError("n must be a multiple of g")
    g0, g1, gspan = _split(n // g, world, rank)
    return ShardPlan("inputs", m, n, q, g, world, rank, g0 * g, g1 * g, gspan * g)


def take_shard(plan: ShardPlan, signs: torch.Tensor, alpha: torch.Tensor):
    """This rank's part of full weights: signs [q][m][n] -> [q][m'][n'] and
    scales [q][n/g][m] -> [q][n'/g][m'] (contiguous copies)."""
    if plan.kind == "rows":
        return (signs[:, plan.lo:plan.hi, :].contiguous(), alpha[:, :, plan.lo:plan.hi].contiguous())
    g0, g1 = plan.lo // plan.g, plan.hi // plan.g
    return (signs[:, :, plan.lo:plan.hi].contiguous(), alpha[:, g0:g1, :].contiguous())


def take_input_slice(plan: ShardPlan, x: torch.Tensor) -> torch.Tensor:
    """The slice of x [batch][n] that an input shard multiplies."""
    return x[:, plan.lo:plan.hi].contiguous() if plan.kind == "inputs" else x


def gather_rows(plan: ShardPlan, y_local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather the row shards' outputs [batch][m'] into y [batch][m].

    Ranges differ by at most one tile; each rank pads its block to the largest
    range so that the collective moves equal blocks, and the padding is dropped."""
    import torch.distributed as dist
    b = y_local.shape[0]
    if b == 1 and plan.m == plan.world * plan.span and y_local.is_contiguous():
        # One batch column, equal ranges: the ranks' rows are consecutive
        # blocks of y as they stand, so they are gathered straight into y.
        out = y_local.new_empty((1, plan.m))
        dist.all_gather_into_tensor(out.view(-1), y_local.view(-1), group=group)
        return out
    block = y_local.new_zeros((plan.span, b))
    block[: y_local.shape[1]] = y_local.t()
    out = y_local.new_empty((plan.world * plan.span, b))
    dist.all_gather_into_tensor(out, block, group=group)
    parts = []
    for r in range(plan.world):
        p = plan_rows(plan.m, plan.n, plan.q, plan.g, plan.world, r)
        parts.append(out[r * plan.span: r * plan.span + (p.hi - p.lo)])
    return torch.cat(parts, 0).t().contiguous()


def reduce_inputs(plan: ShardPlan, y_partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the input shards' partial products [batch][m] over the ranks (in place)."""
    import torch.distributed as dist
    dist.all_reduce(y_partial, op=dist.ReduceOp.SUM, group=group)
    return y_partial


def reduce_scatter_inputs(plan: ShardPlan, y_partial: torch.Tensor, group=None):
    """Sum the partials and leave each rank the rows of ``plan_rows`` for its
    rank: returns (rows plan, y rows [batch][m'])."""
    import torch.distributed as dist
    rows = plan_rows(plan.m, plan.n, plan.q, plan.g, plan.world, plan.rank)
    b = y_partial.shape[0]
    src = y_partial.new_zeros((plan.world * rows.span, b))
    for r in range(plan.world):
        p = plan_rows(plan.m, plan.n, plan.q, plan.g, plan.world, r)
        src[r * rows.span: r * rows.span + (p.hi - p.lo)] = y_partial[:, p.lo:p.hi].t()
    out = y_partial.new_empty((rows.span, b))
    dist.reduce_scatter_tensor(out, src, op=dist.ReduceOp.SUM, group=group)
    return rows, out[: rows.hi - rows.lo].t().contiguous()


class ShardedLinear:
    """One rank's shard of a BCQ linear, on the GPU.

    ``signs`` [q][m'][n'] (+-1, int8) and ``alpha`` [q][n'/g][m'] (fp16) are
    this rank's part (``take_shard``); they are packed once here.  Calling it
    runs ``lutgemm.run`` on the shard and the collective of the plan's kind."""

    def __init__(self, plan: ShardPlan, signs: torch.Tensor, alpha: torch.Tensor, group=None, batch: int = 1):
        from . import lutgemm
        self.plan, self.group = plan, group
        self.m, self.n = plan.local_m, plan.local_n
        if self.m < 1 or self.n < 8:
            raise ValueError("empty shard: use fewer ranks for this matrix")
        self.packed = lutgemm.pack_bcq(signs)
        self.alpha = alpha
        self.workspace = lutgemm.new_workspace(self.m, self.n, batch, plan.q, plan.g, device=signs.device)

    @classmethod
    def from_packed(cls, plan: ShardPlan, packed: torch.Tensor, alpha: torch.Tensor, group=None, batch: int = 1):
        """A shard whose planes are already packed (``lutgemm.pack_bcq`` layout of
        the local [q][m'][n'] matrix); alpha is [q][n'/g][m'] fp16."""
        from . import lutgemm
        self = cls.__new__(cls)
        self.plan, self.group = plan, group
        self.m, self.n = plan.local_m, plan.local_n
        if self.m < 1 or self.n < 8:
            raise ValueError("empty shard: use fewer ranks for this matrix")
        if packed.numel() < lutgemm.packed_bytes(plan.q, self.m, self.n):
            raise ValueError("packed buffer smaller than the shard's packed size")
        self.packed, self.alpha = packed, alpha
        self.workspace = lutgemm.new_workspace(self.m, self.n, batch, plan.q, plan.g, device=packed.device)
        return self

    def local_product(self, x_local: torch.Tensor) -> torch.Tensor:
        from . import lutgemm
        b = x_local.shape[0]
        if lutgemm.workspace_size(self.m, self.n, b, self.plan.q, self.plan.g) > self.workspace.numel():
            self.workspace = lutgemm.new_workspace(self.m, self.n, b, self.plan.q, self.plan.g,
                                                   device=x_local.device)
        return lutgemm.run(self.packed, self.alpha, x_local, self.m, self.n, self.plan.q, self.plan.g,
                           workspace=self.workspace)

    def __call__(self, x: torch.Tensor, gather: bool = True) -> torch.Tensor:
        """x [batch][n] (rows, or inputs with the full x) or [batch][n']
        (inputs, already sliced) -> y [batch][m]; with gather=False a row shard
        returns its own rows [batch][m'] (the hidden slice of a paired block)."""
        p = self.plan
        if p.kind == "rows":
            y = self.local_product(x)
            return gather_rows(p, y, self.group) if gather else y
        xl = x if x.shape[1] == self.n else take_input_slice(p, x)
        return reduce_inputs(p, self.local_product(xl), self.group)


def paired_block(first: ShardedLinear, second: ShardedLinear, x: torch.Tensor, between=None) -> torch.Tensor:
    """y = W2 f(W1 x) with W1 split by rows and W2 by inputs over the same ranks:
    each rank's rows of W1 x are its input slice of W2, so the block makes one
    all-reduce.  ``between`` (elementwise, default identity) maps the fp32
    hidden slice before it is rounded to the fp16 activation W2 reads."""
    if first.plan.kind != "rows" or second.plan.kind != "inputs":
        raise ValueError("the first matrix must be split by rows and the second by inputs")
    if (first.plan.lo, first.plan.hi) != (second.plan.lo, second.plan.hi):
        raise ValueError("the row split of the first matrix must equal the input split of the second")
    h = first(x, gather=False)
    if between is not None:
        h = between(h)
    return second(h.to(torch.float16))


def plan_paired(m1: int, n1: int, m2: int, q: int, g: int, world: int, rank: int):
    """Splits for a paired block W1 [m1][n1] (rows) -> W2 [m2][m1] (inputs): the
    rows of W1 in whole scale groups of W2, so both plans cover the same range."""
    if m1 % g:
        raise ValueError("the hidden size must be a multiple of g")
    second = plan_inputs(m2, m1, q, g, world, rank)
    span = second.span
    first = ShardPlan("rows", m1, n1, q, g, world, rank, second.lo, second.hi, span)
    return first, second
