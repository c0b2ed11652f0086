"""Ulysses sharding on a B200 with a one-rank NCCL group: the all-to-alls around
the path are then the identity and the result must equal the plain path bit for
bit (more ranks need more GPUs than one call here gets; the exchange itself is
covered with gloo ranks on CPU in test_multirank.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from block_sparse_video_rearrange_b200 import rf, synth, ulysses
from tests import parity
from tests.test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    yield dist.group.WORLD
    dist.destroy_process_group()


@pytest.mark.parametrize("name", ["ragged_d128", "tnd_gqa_small"])
def test_one_rank_ulysses_equals_plain_path(nccl_group, name):
    w = SMALL[name]
    bits = synth.generate_qkv(w)
    plain = parity.run_gpu(w, bits)
    att = ulysses.UlyssesAttention(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity,
                                   batch=w.batch, group=nccl_group)
    q, k, v = (parity.to_device(x, w.dtype) for x in bits)
    o = att(q, k, v)
    torch.cuda.synchronize()
    assert np.array_equal(parity.to_bits(o), plain["o"])
