"""Head sharding (one process per GPU, heads split across ranks) gives the
same results as one process running every head.

Two ranks meet over gloo and run their head ranges of one layer through the
unchanged library calls; rank 0 gathers their selection bitmaps, outputs and
gradients and compares them, bit for bit, with a single process's run of all
heads.  On a one-GPU machine both ranks share cuda:0: their kernels are
independent launches that never wait on each other.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import torch.multiprocessing as mp  # noqa: E402

T, H, W, NH, D, MODE, BOX, TAU = 8, 16, 16, 4, 128, 2, (2, 4, 4), 0.4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_heads(heads):
    """bf16 inputs of the layer's heads [h0, h1) -> (sel, out, lse, dq, dk, dv) on the host."""
    import synth
    from synth.video_latents import round_to
    from block_sparse_attention_layer_b200 import LayerShape
    from block_sparse_attention_layer_b200.layer import VMoBALayer
    from tests.gpu_util import to_device
    h0, h1 = heads
    q, k, v = synth.make_qkv(180, 0, T, H, W, NH, D)
    dout = synth.make_dout(180, 0, T * H * W, NH, D)
    xs = [to_device(round_to(np.ascontiguousarray(x[:, h0:h1]), "bf16"), "bf16")
          for x in (q, k, v, dout)]
    L = VMoBALayer(LayerShape(T, H, W, h1 - h0, D, MODE, *BOX, "bf16"))
    L.step(*xs[:3], TAU, dout=xs[3])
    torch.cuda.synchronize()
    return [t.cpu() for t in (L.sel, L.out, L.lse, L.dq, L.dk, L.dv)]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    from block_sparse_attention_layer_b200.sharding import head_range
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        mine = _run_heads(head_range(rank, world, NH))
        parts = [None] * world
        dist.all_gather_object(parts, mine)
        if rank == 0:
            out["parts"] = parts
    finally:
        dist.destroy_process_group()


def test_two_rank_head_shards_equal_one_process():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        parts = out["parts"]
    full = _run_heads((0, NH))
    # heads are dim 0 of sel and lse, dim 1 of out, dq, dk, dv
    for idx, axis in enumerate((0, 1, 0, 1, 1, 1)):
        joined = torch.cat([p[idx] for p in parts], dim=axis)
        assert torch.equal(joined, full[idx]), idx
