"""Seeded synthetic inputs for the ZeRO optimizer-step workloads.

This package is shared by the CUDA harness (tests, bench) and the CPU-oracle
harness. It holds tensor lists, seeds and value recipes and draws numbers; it
holds none of the optimizer step's arithmetic (no reduction, norm, clipping,
loss scaling, AdamW or cast of the step).

Recipe (values are pure functions of seed, stream, step slot and index; see
``zero_synth.h``):
  * master init of a weight / embedding tensor: fp32 of N(0, 0.02) at its flat
    index; norm weights 1; biases 0.
  * replica r gradient at buffer index j, step slot s: N(0, 1e-3), times 8 where
    a per-element Philox word is below 0.001 * 2^32 (only when the workload asks
    for spikes), times the loss scale in force, rounded to the half type.
  * resident workloads: buffer index = flat index, slot = step number t (1-based).
    streaming workloads: the W replica buffers hold one bucket; buffer index =
    flat index - bucket start, slot = (t - 1) % 2.
  * +inf injection: site k of step t picks a flat index in [0, N) and a replica.
  * gradient accumulation (M micro-batches per step, resident workloads): micro-batch k
    of step t draws slot (t-1)*M + k + 1; +inf sites go into the last micro-batch.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libsynth_host.so")
CUDA_LIB = os.path.join(_HERE, "libsynth_cuda.so")

BF16, FP16 = 0, 1
DTYPE_CODE = {"bf16": BF16, "fp16": FP16}

STREAM_INIT = 0
STREAM_GRAD = 1
STREAM_SPIKE = 0x1000
STREAM_INF = 0x2000


def build(cuda: bool = True) -> None:
    """Compile the host fill library (gcc + OpenMP) and the device fill library (nvcc)."""
    subprocess.check_call(
        ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", HOST_LIB,
         os.path.join(_HERE, "synth_host.c")])
    if cuda:
        subprocess.check_call(
            ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
             "-Xcompiler", "-fPIC", "-shared", "-o", CUDA_LIB,
             os.path.join(_HERE, "synth_fill.cu")])


_host = None
_cuda = None


def host_lib():
    global _host
    if _host is None:
        if not os.path.exists(HOST_LIB):
            build(cuda=False)
        lib = ctypes.CDLL(HOST_LIB)
        lib.synth_round_double_host.restype = ctypes.c_uint16
        lib.synth_round_double_host.argtypes = [ctypes.c_double, ctypes.c_int]
        lib.synth_round_double_array_host.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int]
        lib.synth_normal_array_host.argtypes = [
            ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint32,
            ctypes.c_uint32, ctypes.c_uint32, ctypes.c_double]
        lib.synth_fill_grads_host.argtypes = [
            ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint32,
            ctypes.c_uint32, ctypes.c_uint32, ctypes.c_double, ctypes.c_uint32,
            ctypes.c_double, ctypes.c_int]
        lib.synth_fill_master_host.argtypes = [
            ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint32,
            ctypes.c_double]
        lib.synth_inf_site_host.argtypes = [
            ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64,
            ctypes.c_uint32, ctypes.POINTER(ctypes.c_uint64),
            ctypes.POINTER(ctypes.c_uint32)]
        lib.synth_grads_at_host.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32,
            ctypes.c_uint32, ctypes.c_uint32, ctypes.c_double, ctypes.c_uint32,
            ctypes.c_double, ctypes.c_int]
        lib.synth_master_at_host.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32,
            ctypes.c_double]
        _host = lib
    return _host


def cuda_lib():
    global _cuda
    if _cuda is None:
        if not os.path.exists(CUDA_LIB):
            raise RuntimeError(f"{CUDA_LIB} is missing: run synthgen.build()")
        lib = ctypes.CDLL(CUDA_LIB)
        lib.synth_fill_grads_cuda.restype = ctypes.c_int
        lib.synth_fill_grads_cuda.argtypes = [
            ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
            ctypes.c_uint32, ctypes.c_uint32, ctypes.c_double, ctypes.c_uint32,
            ctypes.c_double, ctypes.c_int, ctypes.c_void_p]
        lib.synth_fill_master_cuda.restype = ctypes.c_int
        lib.synth_fill_master_cuda.argtypes = [
            ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
            ctypes.c_double, ctypes.c_void_p]
        _cuda = lib
    return _cuda


def philox(ctr: Sequence[int], key: Sequence[int]) -> List[int]:
    c = (ctypes.c_uint32 * 4)(*ctr)
    k = (ctypes.c_uint32 * 2)(*key)
    o = (ctypes.c_uint32 * 4)()
    host_lib().synth_philox_host(c, k, o)
    return list(o)


def sigma_constant(sigma: float) -> float:
    """c = sigma * sqrt(3) / 2^32: the one double both sides multiply the integer by."""
    return sigma * math.sqrt(3.0) / 4294967296.0


def spike_threshold(frac: float) -> int:
    return int(frac * 4294967296.0) if frac > 0 else 0


# ----------------------------------------------------------------------------
# host fills
# ----------------------------------------------------------------------------

def round_double_to_half(x: np.ndarray, dtype: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    host_lib().synth_round_double_array_host(x.ctypes.data, out.ctypes.data, x.size, dtype)
    return out


def normal_host(j0: int, n: int, seed: int, stream: int, step: int, sigma: float) -> np.ndarray:
    out = np.empty(n, np.float64)
    host_lib().synth_normal_array_host(out.ctypes.data, j0, n, seed, stream, step,
                                       sigma_constant(sigma))
    return out


def grads_host(j0: int, n: int, seed: int, replica: int, slot: int, sigma: float,
               spike_frac: float, scale: float, dtype: int,
               out: Optional[np.ndarray] = None) -> np.ndarray:
    if out is None:
        out = np.empty(n, np.uint16)
    assert out.dtype == np.uint16 and out.size >= n and out.flags.c_contiguous
    host_lib().synth_fill_grads_host(out.ctypes.data, j0, n, seed, replica, slot,
                                     sigma_constant(sigma), spike_threshold(spike_frac),
                                     float(scale), dtype)
    return out


def master_random_host(i0: int, n: int, seed: int, sigma: float,
                       out: Optional[np.ndarray] = None) -> np.ndarray:
    if out is None:
        out = np.empty(n, np.float32)
    host_lib().synth_fill_master_host(out.ctypes.data, i0, n, seed, sigma_constant(sigma))
    return out


def grads_at_host(j: np.ndarray, seed: int, replica: int, slot: int, sigma: float,
                  spike_frac: float, scale: float, dtype: int) -> np.ndarray:
    j = np.ascontiguousarray(j, dtype=np.uint64)
    out = np.empty(j.size, np.uint16)
    host_lib().synth_grads_at_host(out.ctypes.data, j.ctypes.data, j.size, seed, replica, slot,
                                   sigma_constant(sigma), spike_threshold(spike_frac),
                                   float(scale), dtype)
    return out


def master_random_at_host(i: np.ndarray, seed: int, sigma: float) -> np.ndarray:
    i = np.ascontiguousarray(i, dtype=np.uint64)
    out = np.empty(i.size, np.float32)
    host_lib().synth_master_at_host(out.ctypes.data, i.ctypes.data, i.size, seed,
                                    sigma_constant(sigma))
    return out


def inf_site(seed: int, step: int, k: int, n: int, world: int) -> Tuple[int, int]:
    idx = ctypes.c_uint64()
    rep = ctypes.c_uint32()
    host_lib().synth_inf_site_host(seed, step, k, n, world, ctypes.byref(idx), ctypes.byref(rep))
    return int(idx.value), int(rep.value)


# ----------------------------------------------------------------------------
# device fills (harness only: before any timed region)
# ----------------------------------------------------------------------------

def grads_cuda(ptr: int, j0: int, n: int, seed: int, replica: int, slot: int, sigma: float,
               spike_frac: float, scale: float, dtype: int, stream: int) -> None:
    rc = cuda_lib().synth_fill_grads_cuda(ptr, j0, n, seed, replica, slot,
                                          sigma_constant(sigma), spike_threshold(spike_frac),
                                          float(scale), dtype, stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill_grads_cuda failed: cuda error {rc}")


def master_random_cuda(ptr: int, i0: int, n: int, seed: int, sigma: float, stream: int) -> None:
    rc = cuda_lib().synth_fill_master_cuda(ptr, i0, n, seed, sigma_constant(sigma), stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill_master_cuda failed: cuda error {rc}")


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class TensorSpec:
    name: str
    shape: Tuple[int, ...]
    init: str  # "normal" | "ones" | "zeros"

    @property
    def numel(self) -> int:
        n = 1
        for d in self.shape:
            n *= d
        return n


@dataclass
class Workload:
    name: str
    tensors: List[TensorSpec]
    world: int
    bucket: int
    steps: int
    gdtype: str = "bf16"          # gradient and gathered-param half type
    dynamic: bool = False         # dynamic loss scaling
    init_scale_power: int = 16
    loss_scale_window: int = 100
    hysteresis: int = 2
    min_loss_scale: float = 1.0
    align: int = 128
    grad_sigma: float = 1e-3
    init_sigma: float = 0.02
    spike_frac: float = 0.0
    inf_sites: Dict[int, int] = field(default_factory=dict)  # step -> number of +inf sites
    streaming: bool = False
    seed: int = 0
    lr: float = 6e-5
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.01
    max_grad_norm: float = 1.0
    micro_batches: int = 1        # gradient accumulation steps per optimizer step

    @property
    def numels(self) -> List[int]:
        return [t.numel for t in self.tensors]

    @property
    def n(self) -> int:
        return sum(self.numels)

    @property
    def dtype_code(self) -> int:
        return DTYPE_CODE[self.gdtype]

    def slot(self, t: int) -> int:
        return (t - 1) % 2 if self.streaming else t

    def micro_slot(self, t: int, k: int) -> int:
        """Slot of micro-batch k of step t (resident workloads): (t-1)*M + k + 1, which
        is the step number t when there is one micro-batch."""
        return (t - 1) * self.micro_batches + k + 1 if self.micro_batches > 1 else self.slot(t)

    def grad_buffer_len(self, n_pad: int) -> int:
        return min(self.bucket, n_pad) if self.streaming else n_pad

    def inf_sites_at(self, t: int) -> List[Tuple[int, int]]:
        """(flat index, replica) of every +inf planted at step t."""
        return [inf_site(self.seed, t, k, self.n, self.world)
                for k in range(self.inf_sites.get(t, 0))]


def _tiny() -> Workload:
    return Workload("tiny", [TensorSpec("weight", (1024, 1024), "normal")], world=2,
                    bucket=1 << 40, steps=3)


def encoder_tensors(d: int = 4096, ff: int = 2048) -> List[TensorSpec]:
    """nn.TransformerEncoderLayer parameter list in declared order."""
    return [
        TensorSpec("self_attn.in_proj_weight", (3 * d, d), "normal"),
        TensorSpec("self_attn.in_proj_bias", (3 * d,), "zeros"),
        TensorSpec("self_attn.out_proj.weight", (d, d), "normal"),
        TensorSpec("self_attn.out_proj.bias", (d,), "zeros"),
        TensorSpec("linear1.weight", (ff, d), "normal"),
        TensorSpec("linear1.bias", (ff,), "zeros"),
        TensorSpec("linear2.weight", (d, ff), "normal"),
        TensorSpec("linear2.bias", (d,), "zeros"),
        TensorSpec("norm1.weight", (d,), "ones"),
        TensorSpec("norm1.bias", (d,), "zeros"),
        TensorSpec("norm2.weight", (d,), "ones"),
        TensorSpec("norm2.bias", (d,), "zeros"),
    ]


def _enc() -> Workload:
    return Workload("enc", encoder_tensors(), world=4, bucket=500_000_000, steps=10,
                    gdtype="fp16", dynamic=True, inf_sites={3: 5, 7: 5})


def gpt2_medium_tensors(layers: int = 24, d: int = 1024, vocab: int = 50257,
                        ctx: int = 1024, ff: int = 4096) -> List[TensorSpec]:
    ts = [TensorSpec("wte.weight", (vocab, d), "normal"),
          TensorSpec("wpe.weight", (ctx, d), "normal")]
    for i in range(layers):
        p = f"h.{i}."
        ts += [
            TensorSpec(p + "ln_1.weight", (d,), "ones"),
            TensorSpec(p + "ln_1.bias", (d,), "zeros"),
            TensorSpec(p + "attn.c_attn.weight", (d, 3 * d), "normal"),
            TensorSpec(p + "attn.c_attn.bias", (3 * d,), "zeros"),
            TensorSpec(p + "attn.c_proj.weight", (d, d), "normal"),
            TensorSpec(p + "attn.c_proj.bias", (d,), "zeros"),
            TensorSpec(p + "ln_2.weight", (d,), "ones"),
            TensorSpec(p + "ln_2.bias", (d,), "zeros"),
            TensorSpec(p + "mlp.c_fc.weight", (d, ff), "normal"),
            TensorSpec(p + "mlp.c_fc.bias", (ff,), "zeros"),
            TensorSpec(p + "mlp.c_proj.weight", (ff, d), "normal"),
            TensorSpec(p + "mlp.c_proj.bias", (d,), "zeros"),
        ]
    ts += [TensorSpec("ln_f.weight", (d,), "ones"), TensorSpec("ln_f.bias", (d,), "zeros")]
    return ts


def _gpt2() -> Workload:
    return Workload("gpt2", gpt2_medium_tensors(), world=8, bucket=200_000_000, steps=5,
                    spike_frac=0.001)


def llama7b_tensors(layers: int = 32, d: int = 4096, ff: int = 11008,
                    vocab: int = 32000) -> List[TensorSpec]:
    ts = [TensorSpec("model.embed_tokens.weight", (vocab, d), "normal")]
    for i in range(layers):
        p = f"model.layers.{i}."
        ts += [
            TensorSpec(p + "self_attn.q_proj.weight", (d, d), "normal"),
            TensorSpec(p + "self_attn.k_proj.weight", (d, d), "normal"),
            TensorSpec(p + "self_attn.v_proj.weight", (d, d), "normal"),
            TensorSpec(p + "self_attn.o_proj.weight", (d, d), "normal"),
            TensorSpec(p + "mlp.gate_proj.weight", (ff, d), "normal"),
            TensorSpec(p + "mlp.up_proj.weight", (ff, d), "normal"),
            TensorSpec(p + "mlp.down_proj.weight", (d, ff), "normal"),
            TensorSpec(p + "input_layernorm.weight", (d,), "ones"),
            TensorSpec(p + "post_attention_layernorm.weight", (d,), "ones"),
        ]
    ts += [TensorSpec("model.norm.weight", (d,), "ones"),
           TensorSpec("lm_head.weight", (vocab, d), "normal")]
    return ts


def _llama() -> Workload:
    return Workload("llama7b", llama7b_tensors(), world=8, bucket=500_000_000, steps=3,
                    streaming=True)


def sweep(log2n: int, world: int, gdtype: str, steps: int = 10) -> Workload:
    fp16 = gdtype == "fp16"
    return Workload(f"sweep_2^{log2n}_w{world}_{gdtype}",
                    [TensorSpec("flat", (1 << log2n,), "normal")], world=world,
                    bucket=200_000_000, steps=steps, gdtype=gdtype, dynamic=fp16,
                    inf_sites={5: 1} if fp16 else {}, streaming=True)


WORKLOADS = {"tiny": _tiny, "enc": _enc, "gpt2": _gpt2, "llama7b": _llama}


def workload(name: str) -> Workload:
    return WORKLOADS[name]()
