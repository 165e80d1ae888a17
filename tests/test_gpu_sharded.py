"""The head-sharded layer's GPU engine (LibraryEngine) on one rank: with a
world of one no head moves, and the layer's output must be bit-identical to
the single-GPU path on the same heads."""
import datetime
import socket

import pytest
import torch

import datagen

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_one_rank_layer_equals_the_single_gpu_path():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist

    import block_sparse_attention_sba_b200 as sba
    from block_sparse_attention_sba_b200.sharded import HeadShardedAttention, LibraryEngine
    wl = datagen.custom("sharded_small", 1, 5, 5, 19, 21, 128, (2, 8, 8), top_p=(0.6, 0.9),
                        top_k=3, rope_split=(44, 42, 42))
    dev = torch.device("cuda:0")
    q, k, v = datagen.generate(wl, seed=3, device=dev)
    top_p = wl.top_p_per_head()
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube)
    ref = sba.SparseAttention(plan, device=dev)(q, k, v, top_p, wl.top_k)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=dev)
    try:
        eng = LibraryEngine(1, wl.T, wl.Hh, wl.W, wl.d, wl.cube, dev)
        layer = HeadShardedAttention(eng, wl.H, dist.group.WORLD)
        o = layer(q, k, v, top_p, wl.top_k)
        torch.cuda.synchronize()
        assert layer.last_moves == []
        assert torch.equal(o, ref)
    finally:
        dist.destroy_process_group()
