"""Data-parallel weight gradient: token-sharded dW summed over replicas.

The Puro-2B runs train data-parallel (paperlayer.ai summary, section 3
"training recipe", bullet "parallel training": PP = 2 x DP = 12 on 24 GPUs;
arxiv-wiki summary, "Approach" item (2): 24, then 96 GPUs). The
weight gradient dW = dY^T X is a sum over tokens, so the fp32 dW that each
replica computes over its own tokens, summed over the replicas, is the dW of
all tokens. Token shards are whole 128-token groups: the column-wise
(128 x 1) quantisation groups of dY and X then never straddle two replicas,
and a replica's codes and scales are exactly the corresponding slice of the
quantisation of the whole batch.

The local GEMM is the library's fp32 wgrad (fp8bw_gemm_wgrad_f32); the sum
over replicas is an all-reduce of that fp32 buffer through torch.distributed
(NCCL on GPUs).
"""
import torch

GROUP = 128


def token_shard(tokens, world, rank, group=GROUP):
    """[start, stop) of `rank`'s tokens out of `tokens`: contiguous, made of
    whole `group`-token groups (the last group may be short), the groups
    spread as evenly as possible (the first `ngroups % world` ranks take one
    more)."""
    if tokens < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError("bad shard request: tokens=%d world=%d rank=%d"
                         % (tokens, world, rank))
    ngroups = (tokens + group - 1) // group
    base, extra = divmod(ngroups, world)
    g0 = rank * base + min(rank, extra)
    g1 = g0 + base + (1 if rank < extra else 0)
    return min(g0 * group, tokens), min(g1 * group, tokens)


def wgrad_all_reduce(qdy_t, sdy_t, qx_t, sx_t, group=None, stream=None):
    """fp32 dW over the tokens of every replica in `group`.

    qdy_t, sdy_t, qx_t, sx_t: this replica's column-wise quantised dY and X
    (its token shard, see token_shard). Returns the fp32 [n, k] sum over the
    process group of the replicas' local dW; every replica must call this
    with the same n and k. The all-reduce is ordered after the local GEMM on
    `stream` (default: the current stream of the device that holds the
    shards)."""
    import torch.distributed as dist

    from . import ops
    if stream is None:
        stream = torch.cuda.current_stream(qdy_t.device)
    dw = ops.gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, stream=stream)
    if dist.is_available() and dist.is_initialized():
        with torch.cuda.stream(stream):
            dist.all_reduce(dw, op=dist.ReduceOp.SUM, group=group)
    return dw


__all__ = ["GROUP", "token_shard", "wgrad_all_reduce"]
