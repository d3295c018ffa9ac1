"""The sequence-parallel orchestration (top_routed_block_b200.ulysses) with the
library's kernels as the per-rank compute, on one GPU (a one-rank NCCL group: the
all-to-alls are identities and the balancing plan is empty, so nothing waits on
another GPU).  Its output must equal fvattn_route + fvattn_sparse_fwd called
directly, bit for bit."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import workloads as W
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


def test_ulysses_one_rank_equals_direct_calls():
    import top_routed_block_b200 as fv
    from top_routed_block_b200.ulysses import kernel_compute, ulysses_attention
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        w = W.Workload("ulysses_gpu", B=2, H=4, N=2048, d=128, bs=128, p=0.8, dist="structured",
                       grid=(4, 16, 32), head_scale=("uniform", 0.5, 4.0), seed=95)
        Q, K, V = (to_dev(x) for x in W.generate(w))
        counts, attention = kernel_compute(w.p, w.bs)
        O, LSE, st = ulysses_attention(Q, K, V, counts, attention)
        torch.cuda.synchronize()
        r = fv.fvattn_route(Q, K, w.p, w.bs)
        fv.check_status(r.dev_status)
        O_ref, L_ref, stt = fv.fvattn_sparse_fwd(Q, K, V, r.row_ptr, r.col_idx, w.bs, False)
        fv.check_status(stt)
        assert torch.equal(O.view(torch.int16), O_ref.view(torch.int16))
        assert torch.equal(LSE, L_ref)
        assert st.moves == [] and st.loads_before == st.loads_after == [int(r.head_counts.sum().item())]
    finally:
        dist.destroy_process_group()
