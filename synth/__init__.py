"""Seeded synthetic inputs for the W8A8 MoE layer (shared by the oracle side
and the CUDA side; holds none of the layer's arithmetic).

The C generator in ``synth.c`` makes every value a pure function of
(seed, tensor id, element index), so any slice can be regenerated and the two
sides of a parity test always receive identical bytes.

Workload recipes (shapes, seeds, value distributions) follow the workloads
the pages describe: a tiny layer (d=256, 8 experts), a decode step of a
27B-class MoE (batch 32), the matching prefill (batch 32 x 512 prompt tokens,
the "batch 32 / input 512" condition of the gtnt.cn page, section 1.3), a
large sparse layer shaped like the trillion-parameter profile of the
ruibaoantu.com page, section 2 (hidden 8192, 256 experts, top-8), and a
token-count / skew sweep.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libmoe_synth.so")
_lib = None

# Tensor ids: each tensor of a workload draws from its own stream.
TID_X = 1
TID_W_ROUTER = 2
TID_W_GATE = 3
TID_W_UP = 4
TID_W_DOWN = 5
TID_LOGITS = 6
TID_OUTLIERS = 8
TID_BIAS_PERM = 9

CALIB_SEED_OFFSET = 1000
CALIB_TOKENS = 512


def build(force: bool = False) -> str:
    """Compile the generator (gcc, OpenMP) next to this file."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", _SO, src, "-lm"])
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        u64, u32, i32, i64, dbl = (ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int32,
                                   ctypes.c_int64, ctypes.c_double)
        vp = ctypes.c_void_p
        L.synth_normal_f32.argtypes = [u64, u32, u64, u64, dbl, dbl, vp]
        L.synth_uniform_f32.argtypes = [u64, u32, u64, u64, dbl, dbl, vp]
        L.synth_bits_u64.argtypes = [u64, u32, u64, u64, vp]
        L.synth_permutation.argtypes = [u64, u32, i32, vp]
        L.synth_subset.argtypes = [u64, u32, i32, i32, vp]
        L.synth_activations.argtypes = [u64, u32, i64, i64, i32, vp, i32, dbl, i32, vp, vp]
        L.synth_f32_to_bf16.argtypes = [vp, i64, vp]
        for f in (L.synth_normal_f32, L.synth_uniform_f32, L.synth_bits_u64, L.synth_permutation,
                  L.synth_subset, L.synth_activations, L.synth_f32_to_bf16):
            f.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def normal(seed: int, tid: int, shape, std: float = 1.0, mean: float = 0.0, start: int = 0,
           out: np.ndarray | None = None) -> np.ndarray:
    n = int(np.prod(shape))
    if out is None:
        out = np.empty(shape, dtype=np.float32)
    lib().synth_normal_f32(seed, tid, start, n, mean, std, _ptr(out))
    return out


def uniform(seed: int, tid: int, shape, lo: float = 0.0, hi: float = 1.0, start: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    lib().synth_uniform_f32(seed, tid, start, int(np.prod(shape)), lo, hi, _ptr(out))
    return out


def bits(seed: int, tid: int, n: int, start: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    lib().synth_bits_u64(seed, tid, start, n, _ptr(out))
    return out


def permutation(seed: int, tid: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().synth_permutation(seed, tid, n, _ptr(out))
    return out


def subset(seed: int, tid: int, d: int, m: int) -> np.ndarray:
    out = np.empty(max(m, 1), dtype=np.int32)
    lib().synth_subset(seed, tid, d, m, _ptr(out))
    return out[:m].copy()


def activations(seed: int, rows: int, d: int, outliers: np.ndarray, factor: float, bf16: bool,
                row0: int = 0, tid: int = TID_X):
    """X rows [rows][d]: returns (fp32 values, bf16 bits or None)."""
    f32 = np.empty((rows, d), dtype=np.float32)
    b16 = np.empty((rows, d), dtype=np.uint16) if bf16 else None
    oc = np.ascontiguousarray(outliers, dtype=np.int32)
    lib().synth_activations(seed, tid, row0, rows, d, _ptr(oc) if len(oc) else None, len(oc),
                            float(factor), 1 if bf16 else 0, _ptr(f32),
                            _ptr(b16) if b16 is not None else None)
    return f32, b16


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().synth_f32_to_bf16(_ptr(a), a.size, _ptr(out))
    return out


def zipf_bias(seed: int, n_experts: int, s: float = 1.1) -> np.ndarray:
    """Per-expert log-prior of a Zipf(s) popularity: bias_e = -s ln(rank(e)+1),
    with the ranks a seeded permutation of the experts."""
    rank = permutation(seed, TID_BIAS_PERM, n_experts)
    return np.array([-s * math.log(float(r) + 1.0) for r in rank], dtype=np.float64).astype(np.float32)


# --------------------------------------------------------------------------------------
# Workload recipes
# --------------------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    alpha: float
    in_bf16: bool            # activations / output bf16 (else fp32)
    weight_seed: int         # expert weights, outlier channels, calibration draw
    data_seed: int           # X, router weights, router logits, router bias
    outlier_frac: float = 0.0
    outlier_factor: float = 1.0
    fixed_outliers: tuple = ()
    logits_uniform: bool = False   # router logits given directly, U[0,1)
    zipf_s: float = 0.0            # >0: Zipf(s) per-expert router bias
    capacity_factor: float = 0.0   # <=0: no capacity limit
    weight_std: float = 0.02
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def n_outliers(self) -> int:
        if self.fixed_outliers:
            return len(self.fixed_outliers)
        return int(round(self.outlier_frac * self.d))

    def outlier_channels(self) -> np.ndarray:
        if self.fixed_outliers:
            return np.array(self.fixed_outliers, dtype=np.int32)
        return subset(self.weight_seed, TID_OUTLIERS, self.d, self.n_outliers)


WORKLOADS = {
    # tiny layer: T=64, d=256, 8 experts top-2, f=512, fp32, 4 fixed outlier channels x20, alpha 0.5
    "tiny": Workload("tiny", T=64, d=256, E=8, k=2, f=512, alpha=0.5, in_bf16=False,
                     weight_seed=0, data_seed=0, outlier_factor=20.0,
                     fixed_outliers=(0, 64, 128, 192)),
    # decode step of a 27B-class MoE layer: batch 32, d=4096, 64 experts top-4, f=1536
    "decode": Workload("decode", T=32, d=4096, E=64, k=4, f=1536, alpha=0.6, in_bf16=True,
                       weight_seed=1, data_seed=1, outlier_frac=0.005, outlier_factor=30.0,
                       logits_uniform=True),
    # prefill of the same layer (same weights): batch 32 x 512 prompt tokens
    "prefill": Workload("prefill", T=16384, d=4096, E=64, k=4, f=1536, alpha=0.6, in_bf16=True,
                        weight_seed=1, data_seed=2, outlier_frac=0.005, outlier_factor=30.0),
    # large sparse layer: d=8192, 256 experts top-8, f=2048, Zipf(1.1) skew, capacity 1.25
    "large": Workload("large", T=4096, d=8192, E=256, k=8, f=2048, alpha=0.6, in_bf16=True,
                      weight_seed=3, data_seed=3, outlier_frac=0.01, outlier_factor=50.0,
                      zipf_s=1.1, capacity_factor=1.25),
}


def sweep_workloads():
    """Token-count x skew x alpha sweep on the decode layer's shape (and weights):
    seeds 10..41 in the order T, then skew, then alpha."""
    out = []
    seed = 10
    for T in (1, 8, 32, 128, 512, 2048, 8192, 16384):
        for skew in (0.0, 1.1):
            for alpha in (0.5, 0.7):
                out.append(Workload(f"sweep_T{T}_{'zipf' if skew else 'unif'}_a{alpha}", T=T, d=4096,
                                    E=64, k=4, f=1536, alpha=alpha, in_bf16=True, weight_seed=1,
                                    data_seed=seed, outlier_frac=0.005, outlier_factor=30.0,
                                    zipf_s=skew))
                seed += 1
    return out


def custom(name="custom", **kw) -> Workload:
    base = dict(T=64, d=256, E=8, k=2, f=512, alpha=0.5, in_bf16=False, weight_seed=0, data_seed=0,
                outlier_factor=20.0, fixed_outliers=(0, 64, 128, 192))
    base.update(kw)
    return Workload(name, **base)


@dataclass
class LayerWeights:
    w_gate: np.ndarray     # [E][d][f] fp32
    w_up: np.ndarray       # [E][d][f] fp32
    w_down: np.ndarray     # [E][f][d] fp32
    calib_x: np.ndarray    # [CALIB_TOKENS][d] fp32 values (bf16-exact when the layer is bf16)


@dataclass
class LayerData:
    x: np.ndarray                  # [T][d] fp32 values
    x_bits: np.ndarray | None      # [T][d] bf16 bits when the layer is bf16
    w_router: np.ndarray           # [d][E] fp32
    router_logits: np.ndarray | None   # [T][E] fp32 or None
    router_bias: np.ndarray | None     # [E] fp32 or None


def make_weights(w: Workload, experts=None) -> LayerWeights:
    """Expert weights (all experts, or the listed ones in that order) and the
    calibration draw."""
    E, d, f = w.E, w.d, w.f
    ids = list(range(E)) if experts is None else list(experts)
    wg = np.empty((len(ids), d, f), dtype=np.float32)
    wu = np.empty((len(ids), d, f), dtype=np.float32)
    wd = np.empty((len(ids), f, d), dtype=np.float32)
    per = d * f
    for i, e in enumerate(ids):
        normal(w.weight_seed, TID_W_GATE, (d, f), std=w.weight_std, start=e * per, out=wg[i])
        normal(w.weight_seed, TID_W_UP, (d, f), std=w.weight_std, start=e * per, out=wu[i])
        normal(w.weight_seed, TID_W_DOWN, (f, d), std=w.weight_std, start=e * per, out=wd[i])
    calib, _ = activations(w.weight_seed + CALIB_SEED_OFFSET, CALIB_TOKENS, d, w.outlier_channels(),
                           w.outlier_factor, w.in_bf16)
    return LayerWeights(wg, wu, wd, calib)


def make_data(w: Workload, T: int | None = None, row0: int = 0) -> LayerData:
    T = w.T if T is None else T
    x, xb = activations(w.data_seed, T, w.d, w.outlier_channels(), w.outlier_factor, w.in_bf16,
                        row0=row0)
    wr = normal(w.data_seed, TID_W_ROUTER, (w.d, w.E), std=w.weight_std)
    logits = uniform(w.data_seed, TID_LOGITS, (T, w.E), start=row0 * w.E) if w.logits_uniform else None
    bias = zipf_bias(w.data_seed, w.E, w.zipf_s) if w.zipf_s > 0 else None
    return LayerData(x, xb, wr, logits, bias)
