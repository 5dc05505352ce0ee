"""Data-parallel weight gradient (paperlayer.ai summary of the Puro-2B report,
section 3, "parallel training": DP replicas): token shards of whole 128-token
groups, and the identity the decomposition rests on -- the sum over replicas
of the per-shard dW is the dW of all tokens -- checked on the oracle with two
gloo ranks (no GPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synthetic as S
from blockwise_fp8_linear_fp8bw_b200.data_parallel import token_shard


@pytest.mark.parametrize("tokens,world", [(16384, 2), (16384, 8), (1040, 3),
                                          (128, 4), (0, 2), (16400, 96),
                                          (272, 2)])
def test_token_shards_cover_in_whole_groups(tokens, world):
    spans = [token_shard(tokens, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == tokens
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0                        # contiguous, no overlap
    for a0, a1 in spans:
        assert a0 % 128 == 0                   # starts on a group boundary
        assert a1 == tokens or a1 % 128 == 0   # only the last may be short
    sizes = [-(-(a1 - a0) // 128) for a0, a1 in spans]
    assert max(sizes) - min(sizes) <= 1        # groups spread evenly


def test_bad_shard_request():
    with pytest.raises(ValueError):
        token_shard(128, 2, 2)
    with pytest.raises(ValueError):
        token_shard(128, 0, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


M, N, K = 1040, 144, 272


def _inputs():
    dy = S.bf16_normal((M, N), 0, 651, **S.DY_DIST)
    x = S.bf16_normal((M, K), 0, 652, **S.X_DIST)
    return dy, x


def _worker(rank, world, port, out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        dy, x = _inputs()
        t0, t1 = token_shard(M, world, rank)
        q, s = oracle.quantize_colwise(np.ascontiguousarray(dy[t0:t1]))
        qx, sx = oracle.quantize_colwise(np.ascontiguousarray(x[t0:t1]))
        part = oracle.gemm_wgrad(q, s, qx, sx, nthreads=1)
        t = torch.from_numpy(np.ascontiguousarray(part, np.float64))
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        out[rank] = (t.numpy().copy(), (q, s, qx, sx, t0, t1))
    finally:
        dist.destroy_process_group()


def test_sharded_wgrad_sums_to_full_wgrad_on_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    dy, x = _inputs()
    q, s = oracle.quantize_colwise(dy)
    qx, sx = oracle.quantize_colwise(x)
    full, bound = oracle.gemm_wgrad(q, s, qx, sx, with_bound=True)
    for rank in range(world):
        reduced, (rq, rs, rqx, rsx, t0, t1) = res[rank]
        # a shard's codes and scales are the slice of the whole batch's
        g0, g1 = t0 // 128, -(-t1 // 128)
        assert np.array_equal(rq, q[:, t0:t1]) and np.array_equal(rqx, qx[:, t0:t1])
        assert np.array_equal(rs.view(np.uint32), s[g0:g1].view(np.uint32))
        assert np.array_equal(rsx.view(np.uint32), sx[g0:g1].view(np.uint32))
        # the all-reduced sum is the full-batch dW (fp64 rounding only)
        assert np.all(np.abs(reduced - full) <= 1e-12 * (bound + 1e-30))
