"""CPU oracle for the MoonEP hot path -- TEST INFRASTRUCTURE ONLY.

A plain, slow, single-threaded C implementation (``moonep_oracle.c``) of the
plan, dispatch, combine, combine-backward and replica-gradient reduction,
wrapped here with ctypes and numpy.  (The same source is also built with
OpenMP, whose pragmas spread the data steps' token loops over the host's
cores; that build only times a multi-core CPU baseline and never checks
anything.)  Only the test suite, the smoke check
and the benchmark's CPU-baseline / reference legs may import this package;
the product (``load_balancing_moonep_b200``) never does, and this package
never imports the product.

The pages the oracle follows (cited by title and section) are listed in the
header of ``moonep_oracle.c``; each function below names the passage it
implements.
"""
from __future__ import annotations

import ctypes
import struct
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moonep_oracle.c")
_LIB = os.path.join(_HERE, "libmoonep_oracle.so")
# the same source built with OpenMP: its data-step loops run on all host
# cores; used only to time a multi-core CPU baseline, never as the checker
_LIB_OMP = os.path.join(_HERE, "libmoonep_oracle_omp.so")

FLAG_STRICT_BUDGET = 1
FLAG_TRAIN_B_RULE = 2
FLAG_BWD_UNSCALED = 4
FLAG_CASCADE = 8
FLAG_LOCALITY = 16

ST_EXPERT_ID_RANGE = 1
ST_OVERFLOW = 2
ST_STRICT_VIOLATION = 4

INFO_FIELDS = (
    "status", "n_rep", "n_overflow", "n_pieces", "n_receivers",
    "max_rep_per_rank", "n_rep_experts", "n_remote_pairs", "cascade_guard_steps",
    "cascade_guard_slack",
)
INFO_LEN = 16

ERRORS = {0: "ok", 1: "bad argument", 2: "E not divisible by R",
          3: "training budget rule B == E/R violated", 4: "B out of range",
          6: "out of host memory"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False, openmp: bool = True) -> str:
    """Compile the oracle with gcc (plain C11, -O2, no fast-math), and (with
    openmp) the same source with OpenMP for the timed multi-core CPU
    baseline."""
    for lib, extra in ((_LIB, []), (_LIB_OMP, ["-fopenmp"]))[: 2 if openmp else 1]:
        if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(_SRC):
            cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", *extra,
                   "-fPIC", "-shared", "-o", lib, _SRC, "-lm"]
            subprocess.check_call(cmd)
    return _LIB


_lib = None
_lib_omp = None


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def openmp_lib(threads: int = 0):
    """The OpenMP build (data-step loops over all host cores), for timing a
    multi-core CPU baseline only; pass it as ``lib=`` to dispatch, combine
    and reduce_replica_grads.  threads > 0 sets the thread count.  Returns
    (lib, threads in use)."""
    global _lib_omp
    if _lib_omp is None:
        build()
        _lib_omp = _bind(ctypes.CDLL(_LIB_OMP))
    return _lib_omp, int(_lib_omp.or_omp_threads(int(threads)))


def _bind(lib):
    if True:
        lib.or_plan.argtypes = [ctypes.c_void_p] + [ctypes.c_void_p] * 19
        lib.or_plan.restype = ctypes.c_int
        lib.or_check_config.argtypes = [ctypes.c_void_p]
        lib.or_check_config.restype = ctypes.c_int
        lib.or_dispatch.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 2
        lib.or_dispatch.restype = ctypes.c_int
        lib.or_combine.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int64] * 2
        lib.or_combine.restype = ctypes.c_int
        lib.or_combine_backward.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int64] * 2
        lib.or_combine_backward.restype = ctypes.c_int
        lib.or_reduce_replica_grads.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int64] * 3
        lib.or_reduce_replica_grads.restype = ctypes.c_int
        lib.or_prefetch_replicas.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int64] * 3
        lib.or_prefetch_replicas.restype = ctypes.c_int
        lib.or_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.or_f32_to_bf16.restype = ctypes.c_uint16
        lib.or_omp_threads.argtypes = [ctypes.c_int]
        lib.or_omp_threads.restype = ctypes.c_int
        lib.or_set_cascade_capacity.argtypes = [ctypes.c_int32]
        lib.or_set_cascade_capacity.restype = ctypes.c_int32
    return lib


class _Cfg(ctypes.Structure):
    _fields_ = [("R", ctypes.c_int32), ("E", ctypes.c_int32), ("K", ctypes.c_int32),
                ("S", ctypes.c_int32), ("H", ctypes.c_int32), ("B", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


@dataclass(frozen=True)
class Config:
    R: int
    E: int
    K: int
    S: int
    H: int
    B: int
    flags: int = 0

    @property
    def L(self) -> int:
        return self.E // self.R

    @property
    def C(self) -> int:
        return self.S * self.K

    def _c(self) -> _Cfg:
        return _Cfg(self.R, self.E, self.K, self.S, self.H, self.B, self.flags)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int):
    if rc != 0:
        raise OracleError(f"oracle error {rc}: {ERRORS.get(rc, '?')}")


def check_config(cfg: Config) -> int:
    c = cfg._c()
    return _load().or_check_config(ctypes.byref(c))


def f32_to_bf16(x: float) -> int:
    """Round-to-nearest-even fp32 -> bf16 bit pattern (oracle's own routine)."""
    return int(_load().or_f32_to_bf16(ctypes.c_float(x)))


def f32_bits_to_bf16(bits: int) -> int:
    """The same routine on an fp32 given by its bit pattern, passed unchanged
    (a signalling NaN is not quieted on the way in)."""
    f = ctypes.c_float.from_buffer_copy(struct.pack("<I", bits & 0xFFFFFFFF))
    return int(_load().or_f32_to_bf16(f))


def plan(cfg: Config, topk_idx: np.ndarray) -> dict:
    """Steps O1-O8 of the plan (redundant experts planned online from the
    router output so every rank receives exactly S*K slots; MoonEP article,
    'The core idea: dynamic redundant experts').  Returns a dict of numpy
    int32 arrays with the same fields and shapes as the CUDA library's plan."""
    lib = _load()
    R, E, K, S = cfg.R, cfg.E, cfg.K, cfg.S
    topk = np.ascontiguousarray(topk_idx, dtype=np.int32).reshape(R * S, K)
    out = {
        "expert_count": np.zeros(E, np.int32),
        "slot_expert": np.zeros((R, E), np.int32),
        "slot_count": np.zeros((R, E), np.int32),
        "slot_offset": np.zeros((R, E + 1), np.int32),
        "rep_expert": np.zeros(E + R, np.int32),
        "rep_rank": np.zeros(E + R, np.int32),
        "rep_slot": np.zeros(E + R, np.int32),
        "rep_quota": np.zeros(E + R, np.int32),
        "host_ptr": np.zeros(E + 1, np.int32),
        "host_rank": np.zeros(2 * E + R, np.int32),
        "host_slot": np.zeros(2 * E + R, np.int32),
        "host_start": np.zeros(2 * E + R, np.int32),
        "host_quota": np.zeros(2 * E + R, np.int32),
        "host_local": np.zeros(2 * E + R, np.int32),
        "rep_home_list": np.zeros(E, np.int32),
        "dst_pos": np.zeros((R * S, K), np.int32),
        "row_src": np.zeros(R * S * K, np.int32),
        "info": np.zeros(INFO_LEN, np.int32),
    }
    c = cfg._c()
    rc = lib.or_plan(ctypes.byref(c), _p(topk),
                     _p(out["expert_count"]), _p(out["slot_expert"]), _p(out["slot_count"]),
                     _p(out["slot_offset"]), _p(out["rep_expert"]), _p(out["rep_rank"]),
                     _p(out["rep_slot"]), _p(out["rep_quota"]), _p(out["host_ptr"]),
                     _p(out["host_rank"]), _p(out["host_slot"]), _p(out["host_start"]),
                     _p(out["host_quota"]), _p(out["host_local"]), _p(out["rep_home_list"]), _p(out["dst_pos"]),
                     _p(out["row_src"]), _p(out["info"]))
    _check(rc)
    return out


def set_cascade_capacity(c: int) -> int:
    """Lower the replica capacity the relay cascade's guard compares with
    (c <= 0: the plan's E + R - 1); returns the previous setting (0 for the
    default).  For tests that put a cascade step exactly on the limit."""
    return int(_load().or_set_cascade_capacity(int(c)))


def info_dict(p: dict) -> dict:
    return {k: int(p["info"][i]) for i, k in enumerate(INFO_FIELDS)}


def dispatch(cfg: Config, p: dict, hidden_bits: np.ndarray, buf_bits: np.ndarray,
             t0: int = 0, t1: int | None = None, lib=None) -> np.ndarray:
    """Zero-copy permute: hidden row t lands in buffer row dst_pos[t, k] for
    every k (MoonEP article, 'The core idea', zero copy and static shapes).
    hidden_bits: uint16 [R*S, H]; buf_bits: uint16 [R, S*K, H] (written in place)."""
    lib = lib or _load()
    t1 = cfg.R * cfg.S if t1 is None else t1
    assert hidden_bits.dtype == np.uint16 and hidden_bits.flags.c_contiguous
    assert buf_bits.dtype == np.uint16 and buf_bits.flags.c_contiguous
    c = cfg._c()
    _check(lib.or_dispatch(ctypes.byref(c), _p(p["dst_pos"]), _p(p["info"]),
                           _p(hidden_bits), _p(buf_bits), t0, t1))
    return buf_bits


def combine(cfg: Config, p: dict, y_bits: np.ndarray, w: np.ndarray,
            out_bits: np.ndarray | None = None, t0: int = 0, t1: int | None = None,
            lib=None) -> np.ndarray:
    """Weighted unpermute with fp32 fused multiply-add accumulation in k order
    and one bf16 rounding.  y_bits: uint16 [R, S*K, H]; w: float32 [R*S, K]."""
    lib = lib or _load()
    t1 = cfg.R * cfg.S if t1 is None else t1
    if out_bits is None:
        out_bits = np.zeros((cfg.R * cfg.S, cfg.H), np.uint16)
    w = np.ascontiguousarray(w, dtype=np.float32)
    c = cfg._c()
    _check(lib.or_combine(ctypes.byref(c), _p(p["dst_pos"]), _p(p["info"]), _p(y_bits),
                          _p(w), _p(out_bits), t0, t1))
    return out_bits


def combine_backward(cfg: Config, p: dict, dy_bits: np.ndarray, w: np.ndarray,
                     y_bits: np.ndarray, dy_buf_bits: np.ndarray, dw: np.ndarray,
                     t0: int = 0, t1: int | None = None):
    """Backward of the combine: scaled dispatch of dy, and dw[t,k] = <dy[t], y[dst_pos[t,k]]>."""
    lib = _load()
    t1 = cfg.R * cfg.S if t1 is None else t1
    w = np.ascontiguousarray(w, dtype=np.float32)
    assert dw.dtype == np.float32 and dw.flags.c_contiguous
    c = cfg._c()
    _check(lib.or_combine_backward(ctypes.byref(c), _p(p["dst_pos"]), _p(p["info"]),
                                   _p(dy_bits), _p(w), _p(y_bits), _p(dy_buf_bits), _p(dw),
                                   t0, t1))
    return dy_buf_bits, dw


def reduce_replica_grads(cfg: Config, p: dict, reduce_buf: np.ndarray, home_grad: np.ndarray,
                         P: int, i0: int = 0, i1: int | None = None, lib=None):
    """Sum prefetched replicas' fp32 grads into their home expert, ascending
    host rank order, then zero the replica rows (MoonEP article explainer,
    memory tab, training branch).  reduce_buf: f32 [R, B, P]; home_grad: f32 [E, P]."""
    lib = lib or _load()
    i1 = P if i1 is None else i1
    assert reduce_buf.dtype == np.float32 and reduce_buf.flags.c_contiguous
    assert home_grad.dtype == np.float32 and home_grad.flags.c_contiguous
    c = cfg._c()
    _check(lib.or_reduce_replica_grads(ctypes.byref(c), _p(p["host_ptr"]), _p(p["host_rank"]),
                                       _p(p["host_slot"]), _p(p["info"]), _p(reduce_buf),
                                       _p(home_grad), P, i0, i1))
    return reduce_buf, home_grad


def prefetch_replicas(cfg: Config, p: dict, weights_bits: np.ndarray, pool_bits: np.ndarray,
                      P: int, i0: int = 0, i1: int | None = None) -> np.ndarray:
    """Copy each prefetched replica's expert weights into its rank's pool
    slot (MoonEP article explainer, memory tab: duplicated experts are
    prefetched into rows [E, E+B) of the weight pool).  weights_bits: uint16
    [E, P]; pool_bits: uint16 [R, B, P] (written in place).  Returns the
    per-slot weight-row table [R, E] (home e, pool E + r*B + b, overflow e,
    unused -1)."""
    lib = _load()
    i1 = P if i1 is None else i1
    assert weights_bits.dtype == np.uint16 and pool_bits.dtype == np.uint16
    wrow = np.zeros((cfg.R, cfg.E), np.int32)
    c = cfg._c()
    _check(lib.or_prefetch_replicas(ctypes.byref(c), _p(p["slot_expert"]), _p(p["info"]),
                                    _p(weights_bits), _p(pool_bits), _p(wrow), P, i0, i1))
    return wrow
