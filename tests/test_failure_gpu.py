"""Failure detection on the GPU without a fault: every mbarrier wait in the
attention kernel is bounded; the test hook makes one of them run out.  The call
must end with FVATTN_ERR_DEVICE_TIMEOUT recorded in the status word, and the
CUDA context must stay usable (a normal call afterwards is exact)."""
import numpy as np
import pytest
import torch

import workloads as W
from tests.gpu_util import compare_attention, gpu_route, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,bs", [(128, 128), (64, 128), (128, 64)],
                         ids=["d128_bs128", "d64_bs128", "paired_blocks_bs64"])
def test_bounded_wait_times_out_and_context_survives(d, bs, oracle_mod):
    import top_routed_block_b200 as fv
    w = W.Workload("stall", B=1, H=2, N=1024, d=d, bs=bs, p=0.9, dist="structured", grid=(4, 16, 16),
                   head_scale=("uniform", 0.5, 4.0), seed=61)
    Q, K, V = W.generate(w)
    dQ, dK, dV = to_dev(Q), to_dev(K), to_dev(V)
    rp, ci, _ = gpu_route(dQ, dK, w.p, w.bs)
    drp, dci = torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda()
    lib = fv.load_library()
    O = torch.empty_like(dQ)
    L = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    ws = torch.empty(fv.fvattn_fwd_workspace_bytes(w.B, w.H, w.N, w.bs), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.fvattn_test_sparse_fwd_stall(dQ.data_ptr(), dK.data_ptr(), dV.data_ptr(), drp.data_ptr(),
                                          dci.data_ptr(), w.B, w.H, w.N, w.d, w.bs, 0, O.data_ptr(), L.data_ptr(),
                                          ws.data_ptr(), ws.numel(), st.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()                    # returns: the kernel ended on its own
    assert int(st.item()) == fv.FVATTN_ERR_DEVICE_TIMEOUT
    # the context is healthy: a normal call is exact
    O2, L2, st2 = fv.fvattn_sparse_fwd(dQ, dK, dV, drp, dci, w.bs, False)
    fv.check_status(st2)
    tokens = np.arange(w.B * w.H * w.N, dtype=np.int64)
    Oref, Lref = oracle_mod.attn_rows(Q, K, V, w.bs, False, rp, ci, tokens)
    compare_attention(O2, L2, Oref, Lref, tokens, w.d, "after-timeout")
