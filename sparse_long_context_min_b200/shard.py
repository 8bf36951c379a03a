"""One decode step over several GPUs: the kv heads of the batch split over ranks.

Selection is per kv head and the threshold per query head, so nothing inside
the step crosses kv heads.  With one process per GPU, rank r keeps kv heads
[g0, g1) -- their slice of the paged pool and page metadata, and the query
heads of those groups -- and runs its own append, score, select and attend on
them.  The only collective is the gather of the outputs at the end of the
step: every rank contributes its query heads' rows of the [B][H_q][d] output
(torch.distributed.all_gather; NCCL between GPUs).  No rank reads another
rank's memory.

Host logic only: the per-rank step is any callable with the DecodeStep calling
convention (q [B][H_q_local][d], optional new token [B][H_kv_local][1][d]),
normally a DecodeStep over the rank's own pool.
"""
import torch


def kv_head_range(H_kv, world, rank):
    """The kv heads [g0, g1) of `rank`: contiguous blocks, sizes differing by at
    most one, lower ranks taking the larger ones."""
    if not (0 <= rank < world) or world < 1 or H_kv < world:
        raise ValueError("need 0 <= rank < world <= H_kv (got rank %d, world %d, H_kv %d)" % (rank, world, H_kv))
    base, extra = divmod(H_kv, world)
    g0 = rank * base + min(rank, extra)
    return g0, g0 + base + (1 if rank < extra else 0)


def shard(x, dim, g0, g1, per_head=1):
    """The slice of x along `dim` holding kv heads [g0, g1) (per_head entries of
    that dimension per kv head: 1 for kv-head tensors, G for query heads)."""
    return x.narrow(dim, g0 * per_head, (g1 - g0) * per_head)


class HeadShardedStep:
    """A decode step whose kv heads are split over the ranks of `group`.

    step: this rank's step over its kv heads [g0, g1) = kv_head_range(H_kv,
    world, rank) (its pool holds only those heads).  Called with the full
    query [B][H_q][d] (and the full new token [B][H_kv][1][d] when appending),
    it runs `step` on the rank's slice and returns the full output [B][H_q][d]
    gathered from every rank, on every rank.
    """

    def __init__(self, step, H_kv, G, world=1, rank=0, group=None):
        self.step, self.H_kv, self.G = step, H_kv, G
        self.world, self.rank, self.group = world, rank, group
        self.g0, self.g1 = kv_head_range(H_kv, world, rank)
        self.heads = [kv_head_range(H_kv, world, r) for r in range(world)]
        self.most = max(b - a for a, b in self.heads)

    def local_inputs(self, q, k_new=None, v_new=None):
        """This rank's slices of the step's inputs."""
        ql = shard(q, 1, self.g0, self.g1, self.G).contiguous()
        kl = None if k_new is None else shard(k_new, 1, self.g0, self.g1).contiguous()
        vl = None if v_new is None else shard(v_new, 1, self.g0, self.g1).contiguous()
        return ql, kl, vl

    def gather(self, out_local):
        """[B][H_q_local][d] of every rank -> [B][H_q][d] (all ranks)."""
        if self.world == 1:
            return out_local
        B, _, d = out_local.shape
        pad = torch.zeros(B, self.most * self.G, d, dtype=out_local.dtype, device=out_local.device)
        pad[:, :out_local.shape[1]] = out_local
        parts = [torch.empty_like(pad) for _ in range(self.world)]
        torch.distributed.all_gather(parts, pad, group=self.group)
        rows = [parts[r][:, :(b - a) * self.G] for r, (a, b) in enumerate(self.heads)]
        return torch.cat(rows, dim=1)

    def __call__(self, q, k_new=None, v_new=None):
        ql, kl, vl = self.local_inputs(q, k_new, v_new)
        out = self.step(ql, kl, vl) if kl is not None else self.step(ql)
        return self.gather(out)
