"""Verification over a vocabulary split across the ranks of a process group.

"Accelerating Sonar through speculation", section "Draft-target schedule":
the target runs tensor-parallel over a group of ranks.  When its output
projection is split by vocabulary, rank w holds columns [bounds[w],
bounds[w+1]) of every logit row, and no rank has a whole row.  The
verification rule needs whole-row normalisers and one draw per request, so
the ranks exchange a few numbers per row (the kernels are the library's
spec_shard_* calls; the exchanges are NCCL collectives through
torch.distributed):

  1. per-row statistics of the rank's columns         (local kernel)
  2. all-gather of the statistics                     (collective)
  3. the same merge and accept tests on every rank    (local kernel)
  4. fp64 normaliser sums of the draw rows            (local kernel)
  5. all-gather of those                              (collective)
  6. the draw weights' mass in the rank's columns     (local kernel)
  7. all-gather of the masses                         (collective)
  8. the rank whose range holds u * Z draws           (local kernel)
  9. all-reduce (max) of the token                    (collective)
 10. the token written into the outputs               (local kernel)

Greedy verification needs steps 1-3 only.  Every cross-rank sum runs in rank
order inside the kernels, so every rank ends with the same outputs, equal to
the single-GPU calls' under the same rules.

The per-rank computation (`ops`) and the exchanges (`comm`) are objects, so
that the protocol itself can be exercised with other implementations of
either; the defaults are the library's kernels and torch.distributed.
"""
import torch

from . import binding


class TorchComm:
    """The exchanges over a torch.distributed process group (NCCL on GPUs)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.size = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather(self, t):
        parts = [torch.empty_like(t) for _ in range(self.size)]
        self.dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.stack(parts)

    def all_reduce_max(self, t):
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.group)
        return t


class KernelOps:
    """The per-rank steps as the library's kernels (spec_shard_*)."""

    def row_stats(self, target, draft, tokens, lo, hi, temperature):
        return binding.spec_shard_row_stats(target, draft, tokens, lo, hi, temperature)

    def decide(self, max_all, sum_all, probe_all, bounds, tokens, vocab, temperature, seed, offset,
               status):
        return binding.spec_shard_decide(max_all, sum_all, probe_all, bounds, tokens, vocab,
                                         temperature, seed, offset, status=status)

    def decide_greedy(self, max_all, arg_all, tokens, vocab, status):
        return binding.spec_shard_decide_greedy(max_all, arg_all, tokens, vocab, status=status)

    def draw_sums(self, target, draft, lo, hi, temperature, draw, norm_parts):
        return binding.spec_shard_draw_sums(target, draft, lo, hi, temperature, draw, norm_parts)

    def draw_pick(self, target, draft, lo, hi, temperature, draw, norm_parts, mass_parts, me):
        return binding.spec_shard_draw_pick(target, draft, lo, hi, temperature, draw, norm_parts,
                                            mass_parts, me)

    def emit(self, token, draw, out):
        binding.spec_shard_emit(token, draw, out)


class ShardedVerifier:
    """Linear and greedy verification with the vocabulary split over ranks.

    bounds: W + 1 increasing column boundaries (bounds[0] = 0, bounds[W] = V);
    this rank holds columns [bounds[rank], bounds[rank + 1]) of every row, as
    tensors [B][rows][stride] with stride >= its column count."""

    def __init__(self, bounds, rank, comm=None, ops=None, device=None):
        self.bounds = [int(b) for b in bounds]
        if any(b1 <= b0 for b0, b1 in zip(self.bounds[:-1], self.bounds[1:])) or self.bounds[0] != 0:
            raise ValueError("bounds must start at 0 and increase")
        self.W = len(self.bounds) - 1
        self.rank = int(rank)
        if not 0 <= self.rank < self.W:
            raise ValueError("rank outside the bounds")
        self.lo, self.hi = self.bounds[self.rank], self.bounds[self.rank + 1]
        self.comm = comm if comm is not None else TorchComm()
        self.ops = ops if ops is not None else KernelOps()
        self.device = device
        self._bounds_dev = None

    @property
    def vocab(self):
        return self.bounds[-1]

    def _bounds_tensor(self, like):
        if self._bounds_dev is None or self._bounds_dev.device != like.device:
            self._bounds_dev = torch.tensor(self.bounds, dtype=torch.int32, device=like.device)
        return self._bounds_dev

    def verify_linear(self, target, draft, tokens, temperature, seed=0, offset=0, status=None):
        """target [B][k+1][stride], draft [B][k][stride]: this rank's columns.
        Returns (out_tokens [B][k+1], accepted_len [B]), the same on every rank."""
        o, c = self.ops, self.comm
        st = o.row_stats(target, draft, tokens, self.lo, self.hi, temperature)
        max_all = c.all_gather(st["max"])
        sum_all = c.all_gather(st["sum"])
        probe_all = c.all_gather(st["probe"])
        out, acc, draw = o.decide(max_all, sum_all, probe_all, self._bounds_tensor(target), tokens,
                                  self.vocab, temperature, seed, offset, status)
        norm_parts = c.all_gather(o.draw_sums(target, draft, self.lo, self.hi, temperature, draw,
                                              None))
        mass_parts = c.all_gather(o.draw_sums(target, draft, self.lo, self.hi, temperature, draw,
                                              norm_parts))
        token = o.draw_pick(target, draft, self.lo, self.hi, temperature, draw, norm_parts,
                            mass_parts, self.rank)
        c.all_reduce_max(token)
        o.emit(token, draw, out)
        return out, acc

    def verify_greedy(self, target, tokens, status=None):
        """target [B][k+1][stride]: this rank's columns.  Greedy (argmax-match)
        verification; returns (out_tokens, accepted_len) on every rank."""
        o, c = self.ops, self.comm
        st = o.row_stats(target, None, tokens, self.lo, self.hi, 1.0)
        max_all = c.all_gather(st["max"])
        arg_all = c.all_gather(st["arg"])
        return o.decide_greedy(max_all, arg_all, tokens, self.vocab, status)
