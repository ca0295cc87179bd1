"""Head-sharded multi-GPU forward for sequence-sharded inputs.

The distillation recipe the pages describe trains the 14B model with its
token sequence split over GPUs (FastVideo "Distillation" docs, section "Wan2.1
14B Model Sparse-Distill": sequence-parallel size 4).  Block-sparse video
attention cannot run on a sequence shard: a query cube may keep any key cube
of its head, and the cube means need every token of the head.  It is,
however, independent per head.  So each rank trades its token shard of every
head for every token of its own heads (one all-to-all per tensor), runs the
whole single-GPU path (selection, fine pass, optional linear branch) on those
heads with the unchanged library, and trades the output back (one all-to-all).

Layouts (B batches, N = T*H*W tokens, P ranks, heads % P == 0, N % P == 0):
  sequence shard of rank r: [B, N/P, heads, d], tokens [r*N/P, (r+1)*N/P)
  head shard of rank r:     [B, N, heads/P, d], heads  [r*heads/P, (r+1)*heads/P)
The exchange uses torch.distributed (NCCL on GPUs, gloo on CPU); the only
arithmetic is the attention itself, in libvsa.so.  Each byte of q, k, v and of
the output crosses the interconnect at most once per forward.
"""
import torch
import torch.distributed as dist


def _size_rank(group):
    """(ranks, this rank); a single process without a process group is one rank."""
    if not (dist.is_available() and dist.is_initialized()):
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def seq_to_heads(x, group=None):
    """[B, N/P, heads, d] sequence shard -> [B, N, heads/P, d] head shard."""
    P, _ = _size_rank(group)
    if P == 1:
        return x
    B, Nl, heads, d = x.shape
    assert heads % P == 0, f"heads={heads} not divisible by {P} ranks"
    hl = heads // P
    # send[dest] = this rank's tokens of dest's heads
    send = x.reshape(B, Nl, P, hl, d).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)                       # recv[src] = src's tokens of my heads
    dist.all_to_all_single(recv, send, group=group)
    if B == 1:                                          # source-major is token order already
        return recv.view(1, P * Nl, hl, d)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * Nl, hl, d)


def heads_to_seq(y, group=None):
    """[B, N, heads/P, d] head shard -> [B, N/P, heads, d] sequence shard."""
    P, _ = _size_rank(group)
    if P == 1:
        return y
    B, N, hl, d = y.shape
    assert N % P == 0, f"N={N} not divisible by {P} ranks"
    Nl = N // P
    # send[dest] = dest's tokens of my heads
    send = y.reshape(B, P, Nl, hl, d).permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)                       # recv[src] = my tokens of src's heads
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, Nl, P * hl, d)


def exchange_bytes(B, N, heads, d, P, elem=2):
    """Bytes one rank sends per forward: 3 inputs out + 1 output back, each
    the (P-1)/P of its shard that belongs to other ranks."""
    shard = B * (N // P) * heads * d * elem
    return 4 * shard * (P - 1) // P


class SequenceShardedAttention:
    """Forward of block-sparse video attention on sequence-sharded q, k, v:
    seq -> heads all-to-all, the library's select + fine (+ linear) on this
    rank's heads, heads -> seq all-to-all.  One instance per rank; every rank
    calls it with its own shard, in the same order."""

    def __init__(self, B, heads, head_dim, T, H, W, topk, tile=(4, 4, 4), linear=False,
                 group=None, device="cuda"):
        from .ops import BlockSparseVideoAttention
        P, rank = _size_rank(group)
        N = T * H * W
        if heads % P or N % P:
            raise ValueError(f"heads={heads} and N={N} must both be divisible by {P} ranks")
        self.group, self.P, self.rank = group, P, rank
        self.heads, self.N = heads, N
        self.attn = BlockSparseVideoAttention(B, heads // P, head_dim, T, H, W, topk, tile,
                                              linear=linear, device=device)

    def heads_of_rank(self):
        hl = self.heads // self.P
        return range(self.rank * hl, (self.rank + 1) * hl)

    def __call__(self, q_shard, k_shard, v_shard):
        qh, kh, vh = (seq_to_heads(x, self.group) for x in (q_shard, k_shard, v_shard))
        out_heads = self.attn(qh, kh, vh)
        return heads_to_seq(out_heads, self.group)
