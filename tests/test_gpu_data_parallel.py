"""Data-parallel weight gradient on the GPU (one GPU): token shards of the
batch quantised and multiplied separately reproduce the whole batch's
quantisation exactly and, summed, its dW within the GEMM tolerance; the
all-reduce wrapper over a one-rank NCCL group returns the local fp32 dW."""
import datetime
import socket

import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import assert_gemm_close_f32, bf16_np_to_torch

pytestmark = pytest.mark.gpu

M, N, K = 2064, 400, 272      # 17 token groups, the last one short


def _ops():
    from blockwise_fp8_linear_fp8bw_b200 import ops
    return ops


def test_token_shards_reproduce_whole_batch():
    import torch
    from blockwise_fp8_linear_fp8bw_b200.data_parallel import token_shard
    ops = _ops()
    dy = S.bf16_normal((M, N), 0, 661, **S.DY_DIST)
    x = S.bf16_normal((M, K), 0, 662, **S.X_DIST)
    q_all, s_all = ops.quantize_colwise(bf16_np_to_torch(dy))
    qx_all, sx_all = ops.quantize_colwise(bf16_np_to_torch(x))
    total = torch.zeros((N, K), dtype=torch.float32, device="cuda")
    world = 3
    for rank in range(world):
        t0, t1 = token_shard(M, world, rank)
        g0, g1 = t0 // 128, -(-t1 // 128)
        q, s = ops.quantize_colwise(bf16_np_to_torch(dy[t0:t1]))
        qx, sx = ops.quantize_colwise(bf16_np_to_torch(x[t0:t1]))
        assert torch.equal(q, q_all[:, t0:t1]) and torch.equal(qx, qx_all[:, t0:t1])
        assert torch.equal(s.view(torch.int32), s_all[g0:g1].view(torch.int32))
        assert torch.equal(sx.view(torch.int32), sx_all[g0:g1].view(torch.int32))
        total += ops.gemm_wgrad_f32(q, s, qx, sx)
    ops.fp8bw_check_device_error()
    rq, rs = oracle.quantize_colwise(dy)
    rqx, rsx = oracle.quantize_colwise(x)
    acc, bound = oracle.gemm_wgrad(rq, rs, rqx, rsx, with_bound=True)
    assert_gemm_close_f32(total.cpu().numpy(), acc, bound, "sharded wgrad")


def test_wgrad_all_reduce_single_rank_nccl():
    import torch
    import torch.distributed as dist
    from blockwise_fp8_linear_fp8bw_b200.data_parallel import wgrad_all_reduce
    ops = _ops()
    dy = S.bf16_normal((M, N), 0, 663, **S.DY_DIST)
    x = S.bf16_normal((M, K), 0, 664, **S.X_DIST)
    q, s = ops.quantize_colwise(bf16_np_to_torch(dy))
    qx, sx = ops.quantize_colwise(bf16_np_to_torch(x))
    local = ops.gemm_wgrad_f32(q, s, qx, sx)
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port,
                            rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        dw = wgrad_all_reduce(q, s, qx, sx)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(dw, local)
