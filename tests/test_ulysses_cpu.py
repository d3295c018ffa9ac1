"""Sequence-parallel attention with run-time head balancing (FVAttn review,
§1 Key Terms "Ulysses" and "RLB", §3) on gloo ranks on the host: every rank holds
a sequence shard, the all-to-alls regroup heads, the RLB plan moves units between
ranks, and every rank's output shard must equal the oracle's attention of the whole
problem, bit for bit (the per-rank compute here is the oracle itself, so moving a
head changes nothing but where it is computed).  The heads are made uneven so that
the plan moves some of them, and the loads after the moves must not exceed those
before."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W

CASE = W.Workload("ulysses", B=2, H=6, N=768, d=64, bs=64, p=0.7, dist="structured", grid=(3, 16, 16),
                  head_scale=("uniform", 0.3, 6.0), seed=94)   # uneven head groups: the plan moves units


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_fns(w):
    import oracle

    def counts(Q, K):
        r = oracle.route(_bits(Q), _bits(K), w.p, w.bs, nthreads=1)
        return torch.from_numpy(r.head_counts.astype(np.int64))

    def attention(Q, K, V):
        q, k, v = _bits(Q), _bits(K), _bits(V)
        r = oracle.route(q, k, w.p, w.bs, nthreads=1)
        _, U, N, d = q.shape
        tokens = np.arange(U * N, dtype=np.int64)
        O, L = oracle.attn_rows(q, k, v, w.bs, False, r.row_ptr, r.col_idx, tokens, nthreads=1)
        return torch.from_numpy(O.reshape(1, U, N, d)), torch.from_numpy(L.reshape(1, U, N))
    return counts, attention


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from top_routed_block_b200.ulysses import ulysses_attention
        w = CASE
        Q, K, V = (torch.from_numpy(b.view(np.int16)).view(torch.bfloat16) for b in W.generate(w))
        n = w.N // world
        shard = [x[:, :, rank * n:(rank + 1) * n].contiguous() for x in (Q, K, V)]
        counts, attention = _oracle_fns(w)
        O, LSE, st = ulysses_attention(*shard, counts, attention)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), O=O.numpy(), LSE=LSE.numpy(),
                 before=np.array(st.loads_before), after=np.array(st.loads_after), moves=np.array(st.moves),
                 sent=st.units_sent, received=st.units_received)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ulysses_with_rlb_matches_single_process_oracle(world, tmp_path, oracle_mod):
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    w = CASE
    Q, K, V = W.generate(w)
    r = oracle_mod.route(Q, K, w.p, w.bs)
    tokens = np.arange(w.B * w.H * w.N, dtype=np.int64)
    O_ref, L_ref = oracle_mod.attn_rows(Q, K, V, w.bs, False, r.row_ptr, r.col_idx, tokens)
    O_ref = O_ref.reshape(w.B, w.H, w.N, w.d)
    L_ref = L_ref.reshape(w.B, w.H, w.N)
    n = w.N // world
    res = [np.load(tmp_path / f"rank{k}.npz") for k in range(world)]
    for k, z in enumerate(res):
        assert np.array_equal(z["O"], O_ref[:, :, k * n:(k + 1) * n])
        assert np.array_equal(z["LSE"], L_ref[:, :, k * n:(k + 1) * n])
    # every rank saw the same plan; it moved units and did not raise the largest load
    for z in res[1:]:
        assert np.array_equal(z["moves"], res[0]["moves"])
    before, after = res[0]["before"], res[0]["after"]
    assert len(res[0]["moves"]) > 0 and after.max() <= before.max() and after.sum() == before.sum()
    assert sum(int(z["sent"]) for z in res) == sum(int(z["received"]) for z in res)
    # loads before balancing are the per-rank totals of the routed heads of the head groups
    hc = r.head_counts.reshape(w.B, world, w.H // world).sum(axis=(0, 2))
    assert np.array_equal(before, hc)
