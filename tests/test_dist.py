"""Multi-process host logic on CPU (gloo, world size 2): the batch shards
across ranks with no data exchange (each rank's attention on its own batch
rows equals the corresponding rows of the whole-batch result), and the
benchmark's timing reduction takes the maximum over ranks."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    import bench
    import oracle
    from causal_gqa_attention_sm_b200.workloads import custom, make_inputs

    w = custom("dist", B=4, T=40, Hq=6, Hkv=2, D=16, dtype="f32", seed=5)
    full = {n: x.double().numpy() for n, x in make_inputs(w).items()}
    lo, hi = bench.batch_shard(w.B, WORLD, rank)
    mine = {n: x[lo:hi] for n, x in full.items()}
    o, lse = oracle.attn_fwd(mine["q"], mine["k"], mine["v"], w.rope_base, w.causal)
    dq, dk, dv = oracle.attn_bwd(mine["q"], mine["k"], mine["v"], mine["do"], w.rope_base, w.causal)
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), lo=lo, hi=hi, o=o, lse=lse, dq=dq, dk=dk, dv=dv)
    t = bench.max_over_ranks(float(rank + 1) * 1.5, WORLD, device="cpu")
    np.save(os.path.join(out_dir, f"max{rank}.npy"), np.array(t))
    dist.barrier()
    dist.destroy_process_group()


def test_batch_shards_need_no_exchange(tmp_path):
    mp.start_processes(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, start_method="spawn")
    import oracle
    from causal_gqa_attention_sm_b200.workloads import custom, make_inputs

    w = custom("dist", B=4, T=40, Hq=6, Hkv=2, D=16, dtype="f32", seed=5)
    full = {n: x.double().numpy() for n, x in make_inputs(w).items()}
    o, lse = oracle.attn_fwd(full["q"], full["k"], full["v"], w.rope_base, w.causal)
    dq, dk, dv = oracle.attn_bwd(full["q"], full["k"], full["v"], full["do"], w.rope_base, w.causal)
    covered = []
    for r in range(WORLD):
        z = np.load(tmp_path / f"rank{r}.npz")
        lo, hi = int(z["lo"]), int(z["hi"])
        covered += list(range(lo, hi))
        for n, ref in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            np.testing.assert_array_equal(z[n], ref[lo:hi])
        assert float(np.load(tmp_path / f"max{r}.npy")) == 3.0
    assert sorted(covered) == list(range(w.B))
