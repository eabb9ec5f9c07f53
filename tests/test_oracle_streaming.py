"""The oracle's chunked driver for streaming workloads (pass A: per-step scalars from
the gradient stream; pass B: sampled elements through all steps) against the plain
whole-array oracle step on the same inputs laid out in full."""
import numpy as np

import oracle
import synthgen


def _resident_equivalent(wl, steps):
    """Run oracle.step on whole-model replica arrays holding, bucket by bucket, the
    values the streaming recipe puts in the bucket-sized buffers."""
    pl = oracle.plan(wl.numels, wl.world, wl.bucket, wl.align)
    cfg, hp = oracle.workload_cfg(wl)
    st = oracle.state_init(cfg)
    dt = wl.dtype_code
    master = oracle.initial_master(wl, pl.n_pad)
    m = np.zeros(pl.n_pad, np.float32)
    v = np.zeros(pl.n_pad, np.float32)
    R = np.zeros(pl.n_pad, np.float32)
    params = oracle.f32_to_half(master, dt)
    out = []
    for t in range(1, steps + 1):
        scale = oracle.step_grad_scale(wl, st)
        grads = []
        for r in range(wl.world):
            g = np.zeros(pl.n_pad, np.uint16)
            for b in range(pl.n_buckets):
                s, ln = pl.bucket_range(b)
                synthgen.grads_host(0, ln, wl.seed, r, wl.slot(t), wl.grad_sigma, wl.spike_frac,
                                    scale, dt, out=g[s:s + ln])
            grads.append(g)
        for idx, rep in wl.inf_sites_at(t):
            j = idx % wl.bucket
            for b in range(pl.n_buckets):
                s, ln = pl.bucket_range(b)
                if j < ln:
                    grads[rep][s + j] = 0x7C00 if dt == oracle.FP16 else 0x7F80
        sc = oracle.step(grads, dt, wl.bucket, R, master, m, v, params, dt, cfg, hp, st)
        out.append(sc.as_dict())
    return out, dict(master=master, m=m, v=v, params=params, R=R)


def test_streaming_driver_equals_whole_array_step_bf16():
    wl = synthgen.sweep(16, 4, "bf16", steps=4)
    wl.bucket = 10000  # 7 buckets, last one short
    want_sc, want = _resident_equivalent(wl, 4)
    got_sc = oracle.streaming_scalars(wl, chunk=3000)
    for g, w in zip(got_sc, want_sc):
        g = g.as_dict()
        for k in ("overflow", "skipped", "scale_used", "next_scale", "adam_t", "k", "clip_coef"):
            assert g[k] == w[k], k
        assert abs(g["sumsq"] - w["sumsq"]) <= 1e-12 * w["sumsq"]
    idx = np.arange(wl.n, dtype=np.int64)
    got = oracle.streaming_samples(wl, idx, got_sc)
    for k in ("master", "m", "v", "params", "R"):
        assert np.array_equal(got[k], want[k]), k


def test_streaming_driver_fp16_with_overflow():
    wl = synthgen.sweep(15, 4, "fp16", steps=7)
    wl.bucket = 9000
    wl.inf_sites = {5: 1, 6: 1}
    want_sc, want = _resident_equivalent(wl, 7)
    got_sc = oracle.streaming_scalars(wl, chunk=4096)
    assert [s.skipped for s in got_sc] == [w["skipped"] for w in want_sc] == [0, 0, 0, 0, 1, 1, 0]
    assert [s.scale_used for s in got_sc] == [w["scale_used"] for w in want_sc]
    idx = np.arange(wl.n, dtype=np.int64)
    got = oracle.streaming_samples(wl, idx, got_sc)
    for k in ("master", "m", "v", "params"):
        assert np.array_equal(got[k], want[k]), k
