"""Sharded checkpoints: the shard files hold exactly the partitions, a corrupted shard
is refused, a reload (same or another W) restores the unpadded flat state, and a run
continued from a checkpoint equals the run without the interruption."""
import json
import os

import numpy as np
import pytest

import oracle
import synthgen
from zero_sharded_mixed_replica_b200 import checkpoint as ck


def _wl():
    t = synthgen.TensorSpec
    return synthgen.Workload("ck", [t("a", (5000,), "normal"), t("b", (33, 7), "ones"),
                                    t("c", (999,), "normal")], world=4, bucket=1500, steps=4,
                             gdtype="fp16", dynamic=True, align=8, grad_sigma=3e-2,
                             inf_sites={2: 1})


def _fields(wl, ref):
    pl = ref["plan"]
    st = ref["state"]
    return dict(shapes=[t.shape for t in wl.tensors], world_size=wl.world,
                reduce_bucket_size=wl.bucket, align=wl.align, n=pl.n, n_pad=pl.n_pad, p=pl.p,
                dtype=wl.gdtype, scaler_cfg={}, adamw={},
                scaler_state={"scale": st.scale, "cur_hysteresis": st.cur_hysteresis,
                              "iter": st.iter, "last_overflow_iter": st.last_overflow_iter,
                              "adam_t": st.adam_t})


def test_shards_roundtrip_reshard_and_checksum(tmp_path):
    wl = _wl()
    ref = oracle.run_resident(wl, steps=2)
    fields = _fields(wl, ref)
    ck.save_flat(str(tmp_path), fields, ref["master"], ref["m"], ref["v"])
    pl = ref["plan"]
    raw = np.fromfile(os.path.join(tmp_path, "rank00002.bin"), dtype="<f4")
    assert raw.size == 3 * pl.p
    assert np.array_equal(raw[:pl.p], ref["master"][2 * pl.p:3 * pl.p])
    assert np.array_equal(raw[2 * pl.p:], ref["v"][2 * pl.p:3 * pl.p])
    meta, master, m, v = ck.load_flat(str(tmp_path))
    assert meta["scaler_state"]["adam_t"] == ref["state"].adam_t == 1  # step 2 was skipped
    for got, want in ((master, ref["master"]), (m, ref["m"]), (v, ref["v"])):
        assert np.array_equal(got, want[:pl.n])
    # another world size: the same prefix, zero padding, the new partitions
    pl3 = oracle.plan(wl.numels, 3, wl.bucket, wl.align)
    placed = ck.place(master, pl3.n_pad)
    assert np.array_equal(placed[:pl.n], ref["master"][:pl.n]) and not placed[pl.n:].any()
    # a flipped byte is caught
    fn = os.path.join(tmp_path, "rank00001.bin")
    b = bytearray(open(fn, "rb").read())
    b[17] ^= 1
    open(fn, "wb").write(bytes(b))
    with pytest.raises(ValueError, match="checksum"):
        ck.load_flat(str(tmp_path))


def test_continued_run_equals_uninterrupted(tmp_path):
    wl = _wl()
    full = oracle.run_resident(wl, steps=4)
    two = oracle.run_resident(wl, steps=2)
    ck.save_flat(str(tmp_path), _fields(wl, two), two["master"], two["m"], two["v"])
    meta, master, m, v = ck.load_flat(str(tmp_path))
    pl = oracle.plan(wl.numels, wl.world, wl.bucket, wl.align)
    cfg, hp = oracle.workload_cfg(wl)
    st = oracle.State(**meta["scaler_state"])
    master, m, v = (ck.place(a, pl.n_pad) for a in (master, m, v))
    params = oracle.f32_to_half(master, wl.dtype_code)
    R = np.zeros(pl.n_pad, np.float32)
    for t in (3, 4):
        g = oracle.resident_grads(wl, pl.n_pad, t, oracle.step_grad_scale(wl, st))
        oracle.step(g, wl.dtype_code, wl.bucket, R, master, m, v, params, wl.dtype_code,
                    cfg, hp, st)
    for got, want in ((master, full["master"]), (m, full["m"]), (v, full["v"]),
                      (params, full["params"])):
        assert np.array_equal(got, want)
    assert (st.scale, st.adam_t, st.iter) == (full["state"].scale, full["state"].adam_t, 4)


def test_refuses_damaged_or_foreign_directories(tmp_path):
    n, W = 5000, 4
    pl = oracle.plan([n], W, 1000, 1)
    rng = np.random.default_rng(3)
    master, m, v = (rng.standard_normal(pl.n_pad).astype(np.float32) for _ in range(3))
    fields = dict(shapes=[[n]], world_size=W, reduce_bucket_size=1000, align=1, n=pl.n,
                  n_pad=pl.n_pad, p=pl.p, dtype="bf16", scaler_cfg={}, scaler_state={},
                  adamw={})
    d = tmp_path / "ck"
    ck.save_flat(str(d), fields, master, m, v)
    # a shard cut short is refused before anything is read from it
    shard = d / "rank00002.bin"
    data = shard.read_bytes()
    shard.write_bytes(data[:-4])
    with pytest.raises(ValueError, match="bytes, expected"):
        ck.load_flat(str(d))
    shard.write_bytes(data)
    assert np.array_equal(ck.load_flat(str(d))[1], master[:n])
    # zeroed shard: refused by its checksum, read as it is without verification
    shard.write_bytes(bytes(len(data)))
    with pytest.raises(ValueError, match="checksum"):
        ck.load_flat(str(d))
    got = ck.load_flat(str(d), verify=False)[1]
    lo, hi = 2 * pl.p, min(3 * pl.p, n)
    assert not got[lo:hi].any() and np.array_equal(got[:lo], master[:lo])
    # not a checkpoint of this format
    meta = json.loads((d / "meta.json").read_text())
    meta["format"] = "something-else"
    (d / "meta.json").write_text(json.dumps(meta))
    with pytest.raises(ValueError, match="not a"):
        ck.load_flat(str(d))
