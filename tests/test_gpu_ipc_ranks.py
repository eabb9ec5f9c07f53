"""The multi-process step (DistributedZeroStep over CudaRankBackend) with W spawned
processes that share one GPU: every rank maps its peers' gradient and gathered-parameter
buffers with CUDA IPC (offset inside the exporter's allocation included), the bucket
kernel sums the peers' gradients through the mapped pointers in rank order, and the
update stores each rank's half values into every peer's gathered buffer (the fused
all-gather) -- or, unfused, the slices travel through the process group. The ranks
exchange only on the host (a device synchronize, then gloo on CPU tensors), so no
kernel ever waits on another process's kernel. Every rank's partition state and
gathered buffer must equal the oracle's whole-model step, and a ZeRO-3 gather that reads
the peers' partitions through the mappings must rebuild the gathered buffer."""
import datetime
import json
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synthgen

from harness import check_scalars, check_state, half_ulp_distance

pytestmark = pytest.mark.gpu


def _workload(name, world):
    t = synthgen.TensorSpec
    if name == "bf16_ragged":
        return synthgen.Workload(
            "ipc_bf16", [t("a", (100003,), "normal"), t("b", (77, 5), "ones"),
                         t("c", (4097,), "normal")],
            world=world, bucket=30000, steps=3, gdtype="bf16", align=8, grad_sigma=3e-2)
    return synthgen.Workload(
        "ipc_fp16", [t("w", (1 << 18,), "normal"), t("b", (4097,), "zeros")], world=world,
        bucket=50000, steps=4, gdtype="fp16", dynamic=True, align=128, grad_sigma=3e-2,
        inf_sites={2: 1})


def _rank_main(rank, world, port, name, fused, out_dir, ag_bucket=None):
    import torch.distributed as dist

    from synthgen import device as sdev
    import zero_sharded_mixed_replica_b200 as zb
    from zero_sharded_mixed_replica_b200.distributed import CudaRankBackend, DistributedZeroStep

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    torch.cuda.set_device(0)
    wl = _workload(name, world)
    scaler = zb.scaler_cfg(wl.dynamic, wl.init_scale_power, wl.loss_scale_window,
                           wl.hysteresis, wl.min_loss_scale)
    adamw = zb.adamw_cfg(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.max_grad_norm)
    # a small allocation first, so that the buffers below do not start their allocations
    pad = torch.zeros(4096 * (rank + 1), dtype=torch.uint8, device="cuda")
    be = CudaRankBackend([t.shape for t in wl.tensors], wl.bucket, wl.gdtype, rank, world,
                         align=wl.align, scaler=scaler, adamw=adamw, fused_all_gather=fused,
                         host_exchange=True, allgather_bucket_size=ag_bucket)
    s = torch.cuda.current_stream().cuda_stream
    full = torch.zeros(be.n_pad, dtype=torch.float32, device="cuda")
    sdev.init_master(wl, full, s)
    be.master.copy_(full[rank * be.p:(rank + 1) * be.p])
    zb.zero_cast_params(be.plan, full, be.params, wl.gdtype, s)
    offsets = [zb.zero_ipc_get_handle(be.grads)[1], zb.zero_ipc_get_handle(be.params)[1]]
    stepper = DistributedZeroStep(be)
    scale = float(2.0 ** wl.init_scale_power) if wl.dynamic else 1.0
    bits = 0x7C00 if wl.gdtype == "fp16" else 0x7F80
    results = []
    for t in range(1, wl.steps + 1):
        synthgen.grads_cuda(be.grads.data_ptr(), 0, wl.n, wl.seed, rank, wl.micro_slot(t, 0),
                            wl.grad_sigma, wl.spike_frac, scale, wl.dtype_code, s)
        for idx, rep in wl.inf_sites_at(t):
            if rep == rank:
                be.grads.view(torch.int16)[idx] = torch.tensor(bits, dtype=torch.int32).to(torch.int16)
        stepper.step()
        res = be.result()
        results.append(res)
        scale = float(res["next_scale"]) if wl.dynamic else 1.0
    torch.cuda.synchronize()
    # ZeRO-3 gather of every tensor with the peers' partitions read through the mappings
    # (rank q's partition is its slice of its own gathered buffer); must equal this
    # rank's gathered buffer
    parts = [be.peer_params[q] + 2 * q * be.p for q in range(world)]
    gathered = torch.empty(wl.n, dtype=be.params.dtype, device="cuda")
    zb.zero3_gather(be.plan, list(range(len(wl.tensors))), parts, gathered, s)
    torch.cuda.synchronize()
    zero3_ok = bool(torch.equal(gathered.view(torch.int16), be.params[:wl.n].view(torch.int16)))
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), zero3_ok=np.array(zero3_ok),
             master=be.master.cpu().numpy(), m=be.exp_avg.cpu().numpy(),
             v=be.exp_avg_sq.cpu().numpy(), R=be.reduced.cpu().numpy(),
             params=be.params.view(torch.int16).cpu().numpy().view(np.uint16),
             offsets=np.array(offsets), results=np.array(json.dumps(results)))
    dist.barrier()  # nobody touches a peer's memory any more
    be.close()
    dist.barrier()  # every mapping is closed before any rank frees its buffers
    del pad
    dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("world,name,fused,ag_bucket",
                         [(2, "bf16_ragged", True, None), (3, "bf16_ragged", True, None),
                          (2, "fp16_scaler", True, None), (2, "bf16_ragged", False, None),
                          (3, "bf16_ragged", False, 10000)],
                         ids=["w2_bf16_fused", "w3_bf16_fused", "w2_fp16_fused",
                              "w2_bf16_gather_via_group", "w3_bf16_gather_in_buckets"])
def test_ipc_ranks_equal_oracle(world, name, fused, ag_bucket):
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(world, _free_port(), name, fused, d, ag_bucket),
                           nprocs=world, join=True, start_method="spawn")
        ranks = [dict(np.load(os.path.join(d, f"rank{r}.npz"))) for r in range(world)]
    wl = _workload(name, world)
    ref = oracle.run_resident(wl)
    p = ref["plan"].p
    for r, got in enumerate(ranks):
        results = json.loads(str(got["results"]))
        for res, sc in zip(results, ref["scalars"]):
            check_scalars(res, sc)
        sl = slice(r * p, (r + 1) * p)
        assert np.array_equal(got["R"].view(np.uint32), ref["R"][sl].view(np.uint32)), r
        for k in ("master", "m", "v"):
            check_state(k, got[k], ref[k][sl], 1)
        assert half_ulp_distance(got["params"], ref["params"]).max() <= 1, r
        assert bool(got["zero3_ok"]), r
    if name == "fp16_scaler":
        assert [s["skipped"] for s in ref["scalars"]] == [0, 1, 0, 0]
    # the buffers did not start their allocations (the offsets were exercised)
    assert any(int(o) != 0 for got in ranks for o in got["offsets"])
