"""The Ulysses wrapper around the CUDA path on one GPU: a single-rank NCCL group, so
both all-to-alls are exercised (as local exchanges) and the result must equal the
unsharded sparse_attention bit for bit.  Several GPUs are not available to the tests;
the cross-rank exchange is covered by the gloo tests in test_ulysses_multirank.py."""
import os
import socket

import numpy as np
import pytest
import torch

from helpers import to_device
from workloads import make_custom

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_single_rank_nccl_equals_unsharded():
    import datetime

    import torch.distributed as dist

    import video_dit_block_b200 as sba
    from video_dit_block_b200 import ulysses
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        w = make_custom(1, 4, 128, (3, 12, 40), 0.75, seed=29, drop_rate=0.1)
        q, k, v, vl = to_device(w, dev)
        o1, l1 = ulysses.ulysses_attention(q, k, v, vl, 0.75)
        o2, l2, _, _ = sba.sparse_attention(q, k, v, vl, 0.75)
        torch.cuda.synchronize()
        assert sba.device_status() == 0
        assert torch.equal(o1, o2)
        assert torch.equal(l1, l2)
    finally:
        dist.destroy_process_group()
