"""The multi-process ZeRO step (DistributedZeroStep: which rank reduces which work
segments, the rank-ordered exchange of the sums of squares, the all-gather of the
updated half parameters) run on CPU over gloo with W = 2 and 3 spawned ranks. Each rank
drives a CPU backend built on the oracle's functions; the gathered parameters and the
ranks' partition state must equal the single-process oracle step on the same inputs."""
import math
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synthgen


class OracleRankBackend:
    """CPU stand-in for the device side of one rank (test infrastructure)."""

    def __init__(self, wl, rank, world):
        self.wl, self.rank, self.world = wl, rank, world
        self.pl = oracle.plan(wl.numels, world, wl.bucket, wl.align)
        self.n_pad, self.p, self.bucket = self.pl.n_pad, self.pl.p, wl.bucket
        self.cfg, self.hp = oracle.workload_cfg(wl)
        self.state = oracle.state_init(self.cfg)
        self.dt = wl.dtype_code
        full_master = oracle.initial_master(wl, self.n_pad)
        lo = rank * self.p
        self.master = full_master[lo:lo + self.p].copy()
        self.m = np.zeros(self.p, np.float32)
        self.v = np.zeros(self.p, np.float32)
        self.R = np.zeros(self.p, np.float32)
        self.params = oracle.f32_to_half(full_master, self.dt)
        self.grads = np.zeros(self.n_pad, np.uint16)
        self.S_local = 0.0
        self.scalars = []

    def before_peer_reads(self, group):
        # gloo has no 16-bit integer type: carry the half bits as int32
        mine = torch.from_numpy(self.grads.astype(np.int32))
        allg = [torch.empty_like(mine) for _ in range(self.world)]
        dist.all_gather(allg, mine, group=group)
        self.peer_grads = [t.numpy().astype(np.uint16) for t in allg]
        self.S_local = 0.0

    def reduce_segment(self, b):
        bs, bl = self.pl.bucket_range(b)
        lo, hi = max(bs, self.rank * self.p), min(bs + bl, (self.rank + 1) * self.p)
        assert hi > lo
        R = oracle.reduce([np.ascontiguousarray(g[lo:hi]) for g in self.peer_grads], self.dt)
        self.R[lo - self.rank * self.p:hi - self.rank * self.p] = R
        self.S_local = self.S_local + oracle.sumsq(R)

    def local_sumsq(self):
        return torch.tensor([self.S_local], dtype=torch.float64)

    def finalize(self, s_all):
        S = float(s_all[0])
        for q in range(1, self.world):
            S = S + float(s_all[q])
        sc = oracle.finalize(S, not math.isfinite(S), self.cfg, self.hp, self.state)
        self.sc = sc
        self.scalars.append(sc.as_dict())

    def update(self):
        half = np.zeros(self.p, np.uint16)
        lo = self.rank * self.p
        half[:] = self.params[lo:lo + self.p]
        oracle.adamw(self.R, self.master, self.m, self.v, half, self.dt, self.sc)
        self.params[lo:lo + self.p] = half

    def after_update(self, group):
        lo = self.rank * self.p
        mine = torch.from_numpy(self.params[lo:lo + self.p].astype(np.int32))
        out = torch.empty(self.n_pad, dtype=torch.int32)
        dist.all_gather_into_tensor(out, mine, group=group)
        self.params = out.numpy().astype(np.uint16)


def _workloads():
    t = synthgen.TensorSpec
    return {
        "ragged_bf16": synthgen.Workload(
            "dist_bf16", [t("a", (1000,), "normal"), t("b", (3, 7), "ones"), t("c", (1,), "normal"),
                          t("d", (), "zeros"), t("e", (257, 3), "normal")],
            world=0, bucket=37, steps=3, gdtype="bf16", align=1, grad_sigma=3e-2),
        "fp16_scaler": synthgen.Workload(
            "dist_fp16", [t("w", (4096,), "normal"), t("b", (130,), "zeros")], world=0,
            bucket=1000, steps=5, gdtype="fp16", dynamic=True, align=128, grad_sigma=3e-2,
            inf_sites={2: 1, 3: 1}),
    }


def _rank_main(rank, world, port, name, out_dir):
    from zero_sharded_mixed_replica_b200.distributed import DistributedZeroStep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = _workloads()[name]
    wl.world = world
    be = OracleRankBackend(wl, rank, world)
    stepper = DistributedZeroStep(be)
    for t in range(1, wl.steps + 1):
        scale = oracle.step_grad_scale(wl, be.state)
        grads = oracle.resident_grads(wl, be.n_pad, t, scale)
        be.grads = grads[rank].copy()
        stepper.step()
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), master=be.master, m=be.m, v=be.v,
             R=be.R, params=be.params,
             adam_t=np.array([s["adam_t"] for s in be.scalars]),
             skipped=np.array([s["skipped"] for s in be.scalars]),
             scale=np.array([s["scale_used"] for s in be.scalars]),
             norm=np.array([s["norm"] for s in be.scalars]))
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("world,name", [(2, "ragged_bf16"), (3, "ragged_bf16"),
                                        (2, "fp16_scaler")])
def test_distributed_step_equals_single_process(world, name):
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(world, _free_port(), name, d), nprocs=world,
                           join=True, start_method="spawn")
        ranks = [np.load(os.path.join(d, f"rank{r}.npz")) for r in range(world)]
        wl = _workloads()[name]
        wl.world = world
        ref = oracle.run_resident(wl)
        p = ref["plan"].p
        for r, got in enumerate(ranks):
            # every rank holds the same gathered parameters and the same decisions
            assert np.array_equal(got["params"], ref["params"])
            assert list(got["skipped"]) == [s["skipped"] for s in ref["scalars"]]
            assert list(got["scale"]) == [s["scale_used"] for s in ref["scalars"]]
            assert list(got["adam_t"]) == [s["adam_t"] for s in ref["scalars"]]
            for a, b in zip(got["norm"], [s["norm"] for s in ref["scalars"]]):
                assert (math.isnan(a) and math.isnan(b)) or a == b or abs(a - b) <= 1e-12 * abs(b)
            sl = slice(r * p, (r + 1) * p)
            for k in ("master", "m", "v", "R"):
                assert np.array_equal(got[k], ref[k][sl]), (r, k)
        if name == "fp16_scaler":
            assert list(ranks[0]["skipped"]) == [0, 1, 1, 0, 0]


def test_allgather_chunks_cover_the_partition():
    from zero_sharded_mixed_replica_b200.distributed import allgather_chunks
    assert allgather_chunks(0, 5) == []
    assert allgather_chunks(10, None) == [(0, 10)]
    assert allgather_chunks(10, 10) == [(0, 10)] == allgather_chunks(10, 99)
    assert allgather_chunks(10, 3) == [(0, 3), (3, 6), (6, 9), (9, 10)]
    for p in range(1, 60):
        for b in range(1, 70):
            ch = allgather_chunks(p, b)
            assert ch[0][0] == 0 and ch[-1][1] == p
            assert all(a1 == b0 for (_, a1), (b0, _) in zip(ch, ch[1:]))
            assert all(0 < e - s <= b for s, e in ch)
