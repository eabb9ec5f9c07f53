"""Sharded checkpoints of the ZeRO optimizer state, with resharding to another W.

The pages warn that saving a plain `state_dict` loses the shard information and that
the engine's own checkpoint call must be used ([Z2] "大模型分片训练：ZeRO-3策略在PyTorch中的
实现", practice notes). A checkpoint here is a directory:

  meta.json          plan (tensor shapes in declared order, W, reduce_bucket_size,
                     align, n, n_pad, p), half dtype, scaler configuration and state
                     (scale, hysteresis budget, iteration, last overflow, applied
                     steps), AdamW hyperparameters, shard file names and their SHA-256
  rank00000.bin ...  one file per rank: that rank's partition [r*p, (r+1)*p) of the
                     fp32 master weights, then exp_avg, then exp_avg_sq, p
                     little-endian floats each

The gathered half parameters are not stored: they are the round-to-nearest-even cast
of the master weights and are rebuilt on load. The unpadded prefix [0, n) of the flat
space is the same for every W, so loading with another world size (or bucket size or
alignment) re-splits that prefix into the new partitions and zero-fills the new padding.
"""
from __future__ import annotations

import hashlib
import json
import os
from typing import Optional, Sequence, Tuple

import numpy as np

FORMAT = "zero-b200-checkpoint"
VERSION = 1


def _shard_name(r: int) -> str:
    return f"rank{r:05d}.bin"


_CHUNK = 1 << 24  # bytes per hash update / write: large enough to release the GIL well


def _sha256(path: str) -> str:
    h = hashlib.sha256()
    with open(path, "rb") as f:
        for chunk in iter(lambda: f.read(_CHUNK), b""):
            h.update(chunk)
    return h.hexdigest()


def _parallel(fn, items):
    """fn over items on threads (file I/O and hashing release the GIL); in order."""
    items = list(items)
    if len(items) <= 1:
        return [fn(x) for x in items]
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=min(len(items), os.cpu_count() or 1, 16)) as ex:
        return list(ex.map(fn, items))


def write_shard(path: str, rank: int, master: np.ndarray, exp_avg: np.ndarray,
                exp_avg_sq: np.ndarray) -> str:
    """One rank's partition (p elements of each array); returns the file's SHA-256,
    computed over the bytes as they are written (one pass, no copy)."""
    fn = os.path.join(path, _shard_name(rank))
    h = hashlib.sha256()
    with open(fn, "wb") as f:
        for a in (master, exp_avg, exp_avg_sq):
            b = memoryview(np.ascontiguousarray(a, dtype="<f4")).cast("B")
            for i in range(0, len(b), _CHUNK):
                h.update(b[i:i + _CHUNK])
                f.write(b[i:i + _CHUNK])
    return h.hexdigest()


def write_meta(path: str, meta: dict) -> None:
    with open(os.path.join(path, "meta.json"), "w") as f:
        json.dump(meta, f, indent=1, sort_keys=True)


def make_meta(shapes: Sequence[Sequence[int]], world_size: int, reduce_bucket_size: int,
              align: int, n: int, n_pad: int, p: int, dtype: str, scaler_cfg: dict,
              scaler_state: dict, adamw: dict, shard_sha256: Sequence[str]) -> dict:
    return {
        "format": FORMAT, "version": VERSION,
        "shapes": [list(s) for s in shapes], "world_size": world_size,
        "reduce_bucket_size": reduce_bucket_size, "align": align,
        "n": n, "n_pad": n_pad, "p": p, "dtype": dtype,
        "scaler_cfg": scaler_cfg, "scaler_state": scaler_state, "adamw": adamw,
        "shards": [_shard_name(r) for r in range(world_size)],
        "sha256": {_shard_name(r): h for r, h in enumerate(shard_sha256)},
        "shard_layout": "fp32 master, fp32 exp_avg, fp32 exp_avg_sq; p little-endian floats each",
    }


def save_flat(path: str, meta_fields: dict, master: np.ndarray, exp_avg: np.ndarray,
              exp_avg_sq: np.ndarray) -> None:
    """Write all W shards and the metadata from flat n_pad arrays."""
    os.makedirs(path, exist_ok=True)
    W, p = meta_fields["world_size"], meta_fields["p"]
    hashes = _parallel(lambda r: write_shard(path, r, master[r * p:(r + 1) * p],
                                             exp_avg[r * p:(r + 1) * p],
                                             exp_avg_sq[r * p:(r + 1) * p]), range(W))
    write_meta(path, make_meta(shard_sha256=hashes, **meta_fields))


def read_meta(path: str) -> dict:
    with open(os.path.join(path, "meta.json")) as f:
        meta = json.load(f)
    if meta.get("format") != FORMAT or meta.get("version") != VERSION:
        raise ValueError(f"{path}: not a {FORMAT} v{VERSION} checkpoint")
    return meta


def load_flat(path: str, verify: bool = True) -> Tuple[dict, np.ndarray, np.ndarray, np.ndarray]:
    """The unpadded flat state [0, n) of master, exp_avg, exp_avg_sq."""
    meta = read_meta(path)
    W, p, n = meta["world_size"], meta["p"], meta["n"]
    out = [np.empty(W * p, np.float32) for _ in range(3)]

    def read(r):
        # each array's slice is read straight into place and hashed from there
        fn = os.path.join(path, meta["shards"][r])
        if os.path.getsize(fn) != 12 * p:
            raise ValueError(f"{fn}: {os.path.getsize(fn)} bytes, expected {12 * p}")
        h = hashlib.sha256()
        with open(fn, "rb") as f:
            for k in range(3):
                b = memoryview(out[k][r * p:(r + 1) * p]).cast("B")
                for i in range(0, len(b), _CHUNK):
                    got = f.readinto(b[i:i + _CHUNK])
                    if got != len(b[i:i + _CHUNK]):
                        raise ValueError(f"{fn}: short read")
                    if verify:
                        h.update(b[i:i + _CHUNK])
        if verify and h.hexdigest() != meta["sha256"][meta["shards"][r]]:
            raise ValueError(f"{fn}: checksum mismatch")

    _parallel(read, range(W))
    return meta, out[0][:n], out[1][:n], out[2][:n]


def place(flat: np.ndarray, n_pad: int) -> np.ndarray:
    """The unpadded prefix into a zero-padded array of the new plan's n_pad."""
    a = np.zeros(n_pad, np.float32)
    a[:flat.size] = flat
    return a


# ---------------------------------------------------------------------------- device glue

def save(opt, path: str) -> None:
    """Checkpoint a ZeroOptimizer (all W partitions live in one process)."""
    from . import zero_state_read
    st = zero_state_read(opt.workspace, opt._s())
    pl = opt.plan
    sc = {f: getattr(opt.scaler, f) for f, _ in opt.scaler._fields_}
    ad = {f: getattr(opt.adamw, f) for f, _ in opt.adamw._fields_}
    fields = dict(shapes=pl.shapes, world_size=pl.world_size,
                  reduce_bucket_size=pl.bucket_size, align=pl.info.align, n=pl.n,
                  n_pad=pl.n_pad, p=pl.p, dtype=opt.dtype, scaler_cfg=sc, scaler_state=st,
                  adamw=ad)
    save_flat(path, fields, opt.master.cpu().numpy(), opt.exp_avg.cpu().numpy(),
              opt.exp_avg_sq.cpu().numpy())


def load(path: str, world_size: Optional[int] = None, reduce_bucket_size: Optional[int] = None,
         align: Optional[int] = None, device: str = "cuda", verify: bool = True):
    """A ZeroOptimizer restored from a checkpoint, optionally resharded to another
    world size, bucket size or alignment."""
    import torch

    from . import AdamWCfg, ScalerCfg, zero_state_write
    from .optimizer import ZeroOptimizer
    meta, master, m, v = load_flat(path, verify)
    scaler = ScalerCfg(**meta["scaler_cfg"])
    adamw = AdamWCfg(**meta["adamw"])
    opt = ZeroOptimizer(meta["shapes"], world_size or meta["world_size"],
                        reduce_bucket_size or meta["reduce_bucket_size"], meta["dtype"],
                        align or meta["align"], scaler, adamw, device=device)
    n_pad = opt.plan.n_pad
    for dst, src in ((opt.master, master), (opt.exp_avg, m), (opt.exp_avg_sq, v)):
        dst.copy_(torch.from_numpy(place(src, n_pad)))
    zero_state_write(opt.plan, opt.workspace, scaler, meta["scaler_state"], opt._s())
    opt.cast_params()
    return opt
