"""Thin Python binding of the MoonEP C ABI (include/moonep.h).

Argument marshalling only: every step of the plan, permute, unpermute and
reduction runs in the CUDA library ``_lib/libmoonep.so``.  PyTorch supplies
device memory and the current stream.  Importing this module loads the
library and raises ``ImportError`` if it has not been built -- there is no
CPU fallback.

Semantics (MoonEP article, "Moonshot AI Open-Sources MoonEP: A Perfectly
Balanced Expert Parallelism Library for MoE Training", "The core idea:
dynamic redundant experts"): ``plan`` places a few replicas of overloaded
experts so that each of the R simulated ranks receives exactly S*K token
slots; ``dispatch`` writes every (token, k) row straight into its
expert-grouped slot of a static [R, S*K, H] buffer; ``combine`` is the
weighted top-K unpermute; ``reduce_replica_grads`` sums replica gradients
back into their home experts.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libmoonep.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"MoonEP CUDA library not built ({_LIB_PATH} missing): run "
        "`python -m load_balancing_moonep_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)

FLAG_STRICT_BUDGET = 1
FLAG_TRAIN_B_RULE = 2
FLAG_BWD_UNSCALED = 4
FLAG_CASCADE = 8
FLAG_LOCALITY = 16

ST_EXPERT_ID_RANGE = 1
ST_OVERFLOW = 2
ST_STRICT_VIOLATION = 4
ST_ROW_RANGE = 8
ST_WAIT_TIMEOUT = 16
ST_WORKSPACE = 32

INFO_FIELDS = ("status", "n_rep", "n_overflow", "n_pieces", "n_receivers",
               "max_rep_per_rank", "n_rep_experts", "n_remote_pairs", "cascade_guard_steps",
               "cascade_guard_slack")
INFO_LEN = 16

PLAN_FIELDS = ("expert_count", "slot_expert", "slot_count", "slot_offset", "rep_expert", "rep_rank",
               "rep_slot", "rep_quota", "host_ptr", "host_rank", "host_slot", "host_start",
               "host_quota", "rep_home_list", "dst_pos", "row_src", "info", "host_local")

EXPORTED = ("moonep_check_config", "moonep_plan_sizes", "moonep_plan_layout", "moonep_plan",
            "moonep_dispatch", "moonep_combine", "moonep_combine_backward",
            "moonep_reduce_replica_grads", "moonep_error_string", "moonep_abi_version",
            "moonep_plan_noalloc", "moonep_prefetch_replicas", "moonep_status_string",
            "moonep_set_wait_limit", "moonep_ep_sizes", "moonep_ep_count", "moonep_ep_plan",
            "moonep_ep_dispatch", "moonep_ep_combine", "moonep_ep_combine_backward",
            "moonep_ep_reduce_replica_grads", "moonep_ep_prefetch_replicas", "moonep_set_cascade_capacity",
            "moonep_set_plan_path")


class _CConfig(ctypes.Structure):
    _fields_ = [("R", ctypes.c_int32), ("E", ctypes.c_int32), ("K", ctypes.c_int32),
                ("S", ctypes.c_int32), ("H", ctypes.c_int32), ("B", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


class _CPlan(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in PLAN_FIELDS]


_vp = ctypes.c_void_p
_cfgp = ctypes.POINTER(_CConfig)
_planp = ctypes.POINTER(_CPlan)
_lib.moonep_check_config.argtypes = [_cfgp]
_lib.moonep_plan_sizes.argtypes = [_cfgp, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
_lib.moonep_plan_layout.argtypes = [_cfgp, _vp, _planp]
_lib.moonep_plan.argtypes = [_cfgp, _vp, _planp, _vp, _vp]
_lib.moonep_dispatch.argtypes = [_cfgp, _planp, _vp, _vp, _vp]
_lib.moonep_combine.argtypes = [_cfgp, _planp, _vp, _vp, _vp, _vp]
_lib.moonep_combine_backward.argtypes = [_cfgp, _planp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.moonep_reduce_replica_grads.argtypes = [_cfgp, _planp, _vp, _vp, ctypes.c_int64, _vp]
_lib.moonep_plan_noalloc.argtypes = [_cfgp, _vp, _planp, _vp]
_lib.moonep_prefetch_replicas.argtypes = [_cfgp, _planp, _vp, _vp, _vp, ctypes.c_int64, _vp]
_lib.moonep_error_string.argtypes = [ctypes.c_int]
_lib.moonep_error_string.restype = ctypes.c_char_p
_lib.moonep_status_string.argtypes = [ctypes.c_int, ctypes.c_char_p, ctypes.c_size_t]
_lib.moonep_status_string.restype = ctypes.c_char_p
_lib.moonep_abi_version.argtypes = []
_lib.moonep_set_wait_limit.argtypes = [ctypes.c_int]
_lib.moonep_set_cascade_capacity.argtypes = [ctypes.c_int]
_lib.moonep_set_plan_path.argtypes = [ctypes.c_int]
_lib.moonep_ep_sizes.argtypes = [_cfgp, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
_lib.moonep_ep_count.argtypes = [_cfgp, _vp, _vp, _vp, _vp]
_lib.moonep_ep_plan.argtypes = [_cfgp, ctypes.c_int32, _vp, _vp, _planp, _vp, _vp]
_lib.moonep_ep_dispatch.argtypes = [_cfgp, _planp, _vp, _vp, _vp]
_lib.moonep_ep_combine.argtypes = [_cfgp, _planp, _vp, _vp, _vp, _vp]
_lib.moonep_ep_combine_backward.argtypes = [_cfgp, _planp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.moonep_ep_reduce_replica_grads.argtypes = [_cfgp, ctypes.c_int32, _planp, _vp, _vp, ctypes.c_int64, _vp]
_lib.moonep_ep_prefetch_replicas.argtypes = [_cfgp, ctypes.c_int32, _planp, _vp, _vp, _vp, ctypes.c_int64, _vp]
for _f in EXPORTED:
    if _f not in ("moonep_error_string", "moonep_status_string"):
        getattr(_lib, _f).restype = ctypes.c_int

LIB_PATH = _LIB_PATH


class MoonepError(RuntimeError):
    def __init__(self, code: int):
        self.code = code
        super().__init__(f"moonep error {code}: {_lib.moonep_error_string(code).decode()}")


def _check(rc: int):
    if rc != 0:
        raise MoonepError(rc)


@dataclass(frozen=True)
class Config:
    """One MoE layer's shape (moonep_config in moonep.h): R simulated ranks,
    E experts (E % R == 0, L = E/R home experts per rank), top-K, S tokens
    per rank, hidden size H (a multiple of 8), replica budget B per rank, and
    flags: FLAG_STRICT_BUDGET (overflow beyond B is a violation status),
    FLAG_TRAIN_B_RULE (require B == E/R), FLAG_BWD_UNSCALED (combine
    backward dispatches dy unscaled) and FLAG_CASCADE (the planner repairs
    ranks that water-filling leaves over B by a relay cascade)."""
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

    @property
    def tokens(self) -> int:
        return self.R * self.S

    @property
    def pairs(self) -> int:
        return self.R * self.S * self.K

    def c(self) -> _CConfig:
        """The C struct (built once per Config: the calls pass it by reference
        on every plan of a latency-bound layer)."""
        cc = self.__dict__.get("_cc")
        if cc is None:
            cc = _CConfig(self.R, self.E, self.K, self.S, self.H, self.B, self.flags)
            object.__setattr__(self, "_cc", cc)
        return cc


def check_config(cfg: Config) -> int:
    c = cfg.c()
    return _lib.moonep_check_config(ctypes.byref(c))


def plan_sizes(cfg: Config):
    c = cfg.c()
    pb, wb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(_lib.moonep_plan_sizes(ctypes.byref(c), ctypes.byref(pb), ctypes.byref(wb)))
    return pb.value, wb.value


def ep_sizes(cfg: Config):
    """(plan bytes, workspace bytes) of one rank in expert parallelism."""
    c = cfg.c()
    pb, wb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(_lib.moonep_ep_sizes(ctypes.byref(c), ctypes.byref(pb), ctypes.byref(wb)))
    return pb.value, wb.value


class Plan:
    """Device plan block plus the planner workspace, with int32 views of
    every field (shapes as in moonep.h).  ep=True sizes the workspace for
    one rank of expert parallelism (moonep_ep_count / moonep_ep_plan)."""

    def __init__(self, cfg: Config, device=None, ep: bool = False):
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.cfg = cfg
        self.ep = ep
        pb, wb = ep_sizes(cfg) if ep else plan_sizes(cfg)
        self.block = torch.zeros(pb, dtype=torch.uint8, device=device)
        # zero-filled once; every plan call leaves it ready for the next call
        # with this configuration
        self.workspace = torch.zeros(max(wb, 256), dtype=torch.uint8, device=device)
        self.c_plan = _CPlan()
        c = cfg.c()
        _check(_lib.moonep_plan_layout(ctypes.byref(c), self.block.data_ptr(), ctypes.byref(self.c_plan)))
        R, E, K, S = cfg.R, cfg.E, cfg.K, cfg.S
        shapes = {
            "expert_count": (E,), "slot_expert": (R, E), "slot_count": (R, E),
            "slot_offset": (R, E + 1), "rep_expert": (E + R,), "rep_rank": (E + R,),
            "rep_slot": (E + R,), "rep_quota": (E + R,), "host_ptr": (E + 1,),
            "host_rank": (2 * E + R,), "host_slot": (2 * E + R,), "host_start": (2 * E + R,),
            "host_quota": (2 * E + R,), "rep_home_list": (E,), "dst_pos": (R * S, K),
            "row_src": (R * S * K,), "info": (INFO_LEN,), "host_local": (2 * E + R,),
        }
        base = self.block.data_ptr()
        i32 = self.block.view(torch.int32) if pb % 4 == 0 else None
        self.fields = {}
        for f in PLAN_FIELDS:
            off = (getattr(self.c_plan, f) - base) // 4
            n = 1
            for s in shapes[f]:
                n *= s
            self.fields[f] = i32[off:off + n].view(shapes[f])

    def __getattr__(self, name):
        f = self.__dict__.get("fields")
        if f is not None and name in f:
            return f[name]
        raise AttributeError(name)

    def info(self) -> dict:
        """Status and statistics (synchronises with the device)."""
        v = self.fields["info"].cpu().tolist()
        return {k: v[i] for i, k in enumerate(INFO_FIELDS)}

    @property
    def dst_pos_local(self) -> torch.Tensor:
        """Expert parallelism: the global buffer rows of this rank's own
        pairs [S, K] (the first S*K entries of dst_pos)."""
        c = self.cfg
        return self.fields["dst_pos"].view(-1)[: c.S * c.K].view(c.S, c.K)

    def to_numpy(self) -> dict:
        return {k: v.cpu().numpy() for k, v in self.fields.items()}


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _need(t: torch.Tensor, dtype, shape, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def plan(cfg: Config, topk_idx: torch.Tensor, out: Plan | None = None, stream=None) -> Plan:
    """Plan replicas and buffer rows for int32 top-K ids [R*S, K] (two
    kernels, no host synchronisation)."""
    _need(topk_idx, torch.int32, (cfg.tokens, cfg.K), "topk_idx")
    p = Plan(cfg, topk_idx.device) if out is None else out
    c = cfg.c()
    _check(_lib.moonep_plan(ctypes.byref(c), topk_idx.data_ptr(), ctypes.byref(p.c_plan),
                            p.workspace.data_ptr(), _stream(stream)))
    return p


NOALLOC_WORKSPACE_BYTES = 4 << 20


def plan_noalloc(cfg: Config, topk_idx: torch.Tensor, out: Plan, stream=None) -> Plan:
    """Same plan as ``plan`` without using the workspace of ``out``: the
    library's fixed device array serves as scratch space instead.  For
    callers that cannot allocate device memory (a runtime that owns every
    allocation, a hot path that must not call cudaMalloc).  ``out`` still
    provides the plan arrays.  Calls share one array per device, so calls
    that overlap on the GPU race; the first call on a device should come
    before any stream capture."""
    _need(topk_idx, torch.int32, (cfg.tokens, cfg.K), "topk_idx")
    c = cfg.c()
    _check(_lib.moonep_plan_noalloc(ctypes.byref(c), topk_idx.data_ptr(), ctypes.byref(out.c_plan),
                                    _stream(stream)))
    return out


def dispatch(cfg: Config, p: Plan, hidden: torch.Tensor, buf: torch.Tensor | None = None,
             stream=None) -> torch.Tensor:
    """buf[dst_pos[t, k]] = hidden[t]; returns the static [R, S*K, H] bf16 buffer."""
    _need(hidden, torch.bfloat16, (cfg.tokens, cfg.H), "hidden")
    if buf is None:
        buf = torch.empty((cfg.R, cfg.C, cfg.H), dtype=torch.bfloat16, device=hidden.device)
    _need(buf, torch.bfloat16, (cfg.R, cfg.C, cfg.H), "buf")
    c = cfg.c()
    _check(_lib.moonep_dispatch(ctypes.byref(c), ctypes.byref(p.c_plan), hidden.data_ptr(),
                                buf.data_ptr(), _stream(stream)))
    return buf


def combine(cfg: Config, p: Plan, y: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None,
            stream=None) -> torch.Tensor:
    """out[t] = bf16(sum_k w[t,k] * y[dst_pos[t,k]]), fp32 FMA in k order."""
    _need(y, torch.bfloat16, (cfg.R, cfg.C, cfg.H), "y")
    _need(w, torch.float32, (cfg.tokens, cfg.K), "w")
    if out is None:
        out = torch.empty((cfg.tokens, cfg.H), dtype=torch.bfloat16, device=y.device)
    _need(out, torch.bfloat16, (cfg.tokens, cfg.H), "out")
    c = cfg.c()
    _check(_lib.moonep_combine(ctypes.byref(c), ctypes.byref(p.c_plan), y.data_ptr(), w.data_ptr(),
                               out.data_ptr(), _stream(stream)))
    return out


def combine_backward(cfg: Config, p: Plan, dy: torch.Tensor, w: torch.Tensor, y: torch.Tensor,
                     dy_buf: torch.Tensor | None = None, dw: torch.Tensor | None = None, stream=None):
    """Returns (dy_buf [R, S*K, H] bf16, dw [R*S, K] fp32)."""
    _need(dy, torch.bfloat16, (cfg.tokens, cfg.H), "dy")
    _need(w, torch.float32, (cfg.tokens, cfg.K), "w")
    _need(y, torch.bfloat16, (cfg.R, cfg.C, cfg.H), "y")
    if dy_buf is None:
        dy_buf = torch.empty((cfg.R, cfg.C, cfg.H), dtype=torch.bfloat16, device=dy.device)
    if dw is None:
        dw = torch.empty((cfg.tokens, cfg.K), dtype=torch.float32, device=dy.device)
    _need(dy_buf, torch.bfloat16, (cfg.R, cfg.C, cfg.H), "dy_buf")
    _need(dw, torch.float32, (cfg.tokens, cfg.K), "dw")
    c = cfg.c()
    _check(_lib.moonep_combine_backward(ctypes.byref(c), ctypes.byref(p.c_plan), dy.data_ptr(),
                                        w.data_ptr(), y.data_ptr(), dy_buf.data_ptr(), dw.data_ptr(),
                                        _stream(stream)))
    return dy_buf, dw


def reduce_replica_grads(cfg: Config, p: Plan, reduce_buf: torch.Tensor, home_grad: torch.Tensor,
                         stream=None):
    """home_grad[e] += replica grads of e (ascending rank), then zero them.
    reduce_buf: fp32 [R, B, P]; home_grad: fp32 [E, P]."""
    P = home_grad.shape[-1]
    _need(home_grad, torch.float32, (cfg.E, P), "home_grad")
    _need(reduce_buf, torch.float32, (cfg.R, cfg.B, P), "reduce_buf")
    c = cfg.c()
    _check(_lib.moonep_reduce_replica_grads(ctypes.byref(c), ctypes.byref(p.c_plan),
                                            reduce_buf.data_ptr() if reduce_buf.numel() else None,
                                            home_grad.data_ptr(), P, _stream(stream)))
    return home_grad


def prefetch_replicas(cfg: Config, p: Plan, weights: torch.Tensor, pool: torch.Tensor,
                      slot_wrow: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Copy each prefetched replica's expert weights (bf16 [E, P]) into its
    rank's pool slot (bf16 [R, B, P]) and return the per-slot weight-row
    table (int32 [R, E]: home e, pool E + r*B + b, overflow e, unused -1)."""
    P = weights.shape[-1]
    _need(weights, torch.bfloat16, (cfg.E, P), "weights")
    _need(pool, torch.bfloat16, (cfg.R, cfg.B, P), "pool")
    if slot_wrow is None:
        slot_wrow = torch.empty((cfg.R, cfg.E), dtype=torch.int32, device=weights.device)
    _need(slot_wrow, torch.int32, (cfg.R, cfg.E), "slot_wrow")
    c = cfg.c()
    _check(_lib.moonep_prefetch_replicas(ctypes.byref(c), ctypes.byref(p.c_plan), weights.data_ptr(),
                                         pool.data_ptr() if pool.numel() else None, slot_wrow.data_ptr(),
                                         P, _stream(stream)))
    return slot_wrow


# ------------------------------------------------- expert parallelism

def pointer_array(tensors, device=None) -> torch.Tensor:
    """A device int64 array of the tensors' data pointers (index = rank): the
    form in which the expert-parallel calls take the R ranks' buffers.  The
    tensors may live in other GPUs' memory mapped into this process (peer
    memory) or, on one GPU, be R separate allocations."""
    dev = device if device is not None else tensors[0].device
    return torch.tensor([t.data_ptr() if t is not None else 0 for t in tensors], dtype=torch.int64, device=dev)


def ep_count(cfg: Config, topk_local: torch.Tensor, p: Plan, counts_row: torch.Tensor | None = None,
             stream=None) -> torch.Tensor:
    """This rank's counts row [E + 1] int32 (pairs per expert, then invalid ids)."""
    _need(topk_local, torch.int32, (cfg.S, cfg.K), "topk_local")
    if counts_row is None:
        counts_row = torch.empty(cfg.E + 1, dtype=torch.int32, device=topk_local.device)
    _need(counts_row, torch.int32, (cfg.E + 1,), "counts_row")
    c = cfg.c()
    _check(_lib.moonep_ep_count(ctypes.byref(c), topk_local.data_ptr(), counts_row.data_ptr(),
                                p.workspace.data_ptr(), _stream(stream)))
    return counts_row


def ep_gather_counts(counts_row: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's counts row into [R, E + 1] (row r from rank r)
    with torch.distributed: 4 (E + 1) bytes per rank, the one collective of
    an expert-parallel layer's plan."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    n = counts_row.numel()
    out = torch.empty(world * n, dtype=counts_row.dtype, device=counts_row.device)
    dist.all_gather_into_tensor(out, counts_row.contiguous().view(-1), group=group)
    return out.view(world, n)


def ep_plan(cfg: Config, rank: int, topk_local: torch.Tensor, counts_all: torch.Tensor, p: Plan,
            stream=None) -> Plan:
    """Every rank's identical plan tables from the gathered counts, and the
    global rows of this rank's own pairs (p.dst_pos_local)."""
    _need(topk_local, torch.int32, (cfg.S, cfg.K), "topk_local")
    _need(counts_all, torch.int32, (cfg.R, cfg.E + 1), "counts_all")
    c = cfg.c()
    _check(_lib.moonep_ep_plan(ctypes.byref(c), int(rank), topk_local.data_ptr(), counts_all.data_ptr(),
                               ctypes.byref(p.c_plan), p.workspace.data_ptr(), _stream(stream)))
    return p


def _need_ptrs(t: torch.Tensor, cfg: Config, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.int64 or t.numel() != cfg.R:
        raise ValueError(f"{name} must be a CUDA int64 tensor of {cfg.R} pointers (see pointer_array)")


def ep_dispatch(cfg: Config, p: Plan, hidden_local: torch.Tensor, buf_ptrs: torch.Tensor, stream=None):
    """Write this rank's token rows into every rank's [S*K, H] buffer."""
    _need(hidden_local, torch.bfloat16, (cfg.S, cfg.H), "hidden_local")
    _need_ptrs(buf_ptrs, cfg, "buf_ptrs")
    c = cfg.c()
    _check(_lib.moonep_ep_dispatch(ctypes.byref(c), ctypes.byref(p.c_plan), hidden_local.data_ptr(),
                                   buf_ptrs.data_ptr(), _stream(stream)))


def ep_combine(cfg: Config, p: Plan, y_ptrs: torch.Tensor, w_local: torch.Tensor,
               out_local: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """This rank's tokens' weighted sum of their K expert-output rows, read
    from every rank's buffer."""
    _need_ptrs(y_ptrs, cfg, "y_ptrs")
    _need(w_local, torch.float32, (cfg.S, cfg.K), "w_local")
    if out_local is None:
        out_local = torch.empty((cfg.S, cfg.H), dtype=torch.bfloat16, device=w_local.device)
    _need(out_local, torch.bfloat16, (cfg.S, cfg.H), "out_local")
    c = cfg.c()
    _check(_lib.moonep_ep_combine(ctypes.byref(c), ctypes.byref(p.c_plan), y_ptrs.data_ptr(), w_local.data_ptr(),
                                  out_local.data_ptr(), _stream(stream)))
    return out_local


def ep_combine_backward(cfg: Config, p: Plan, dy_local: torch.Tensor, w_local: torch.Tensor,
                        y_ptrs: torch.Tensor, dy_buf_ptrs: torch.Tensor, dw_local: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """Backward of ep_combine: scaled dy rows into every rank's dy buffer,
    and this rank's dw [S, K]."""
    _need(dy_local, torch.bfloat16, (cfg.S, cfg.H), "dy_local")
    _need(w_local, torch.float32, (cfg.S, cfg.K), "w_local")
    _need_ptrs(y_ptrs, cfg, "y_ptrs")
    _need_ptrs(dy_buf_ptrs, cfg, "dy_buf_ptrs")
    if dw_local is None:
        dw_local = torch.empty((cfg.S, cfg.K), dtype=torch.float32, device=dy_local.device)
    _need(dw_local, torch.float32, (cfg.S, cfg.K), "dw_local")
    c = cfg.c()
    _check(_lib.moonep_ep_combine_backward(ctypes.byref(c), ctypes.byref(p.c_plan), dy_local.data_ptr(),
                                           w_local.data_ptr(), y_ptrs.data_ptr(), dy_buf_ptrs.data_ptr(),
                                           dw_local.data_ptr(), _stream(stream)))
    return dw_local


def ep_reduce_replica_grads(cfg: Config, rank: int, p: Plan, reduce_buf_ptrs: torch.Tensor,
                            home_grad_local: torch.Tensor, stream=None) -> torch.Tensor:
    """On home rank `rank`: pull its experts' replica gradient rows from every
    rank's [B, P] reduce buffer into home_grad_local [L, P], zeroing them."""
    P = home_grad_local.shape[-1]
    _need(home_grad_local, torch.float32, (cfg.L, P), "home_grad_local")
    _need_ptrs(reduce_buf_ptrs, cfg, "reduce_buf_ptrs")
    c = cfg.c()
    _check(_lib.moonep_ep_reduce_replica_grads(ctypes.byref(c), int(rank), ctypes.byref(p.c_plan),
                                               reduce_buf_ptrs.data_ptr(), home_grad_local.data_ptr(), P,
                                               _stream(stream)))
    return home_grad_local


def ep_prefetch_replicas(cfg: Config, rank: int, p: Plan, weight_ptrs: torch.Tensor, pool_local: torch.Tensor,
                         slot_wrow_local: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """On rank `rank`: pull each prefetched replica's weight row ([L, P] bf16
    home weights of every rank, through weight_ptrs) into pool_local [B, P];
    returns the local slot table [E] (home s, pool L + b, overflow L + B + e
    read through from the home rank, unused -1)."""
    P = pool_local.shape[-1]
    _need(pool_local, torch.bfloat16, (cfg.B, P), "pool_local")
    _need_ptrs(weight_ptrs, cfg, "weight_ptrs")
    if slot_wrow_local is None:
        slot_wrow_local = torch.empty(cfg.E, dtype=torch.int32, device=pool_local.device)
    _need(slot_wrow_local, torch.int32, (cfg.E,), "slot_wrow_local")
    c = cfg.c()
    _check(_lib.moonep_ep_prefetch_replicas(ctypes.byref(c), int(rank), ctypes.byref(p.c_plan),
                                            weight_ptrs.data_ptr(),
                                            pool_local.data_ptr() if pool_local.numel() else None,
                                            slot_wrow_local.data_ptr(), P, _stream(stream)))
    return slot_wrow_local


def views(cfg: Config, p: Plan, buf: torch.Tensor):
    """Debug convenience: per-(rank, slot) (expert, view) lists of the
    buffer.  Synchronises the host (slicing needs host offsets); the hot path
    hands the device-side slot_offset/slot_count to a grouped GEMM instead."""
    so = p.slot_offset.cpu()
    se = p.slot_expert.cpu()
    out = []
    for r in range(cfg.R):
        row = []
        for s in range(cfg.E):
            e = int(se[r, s])
            if e < 0:
                break
            row.append((e, buf[r, int(so[r, s]):int(so[r, s + 1])]))
        out.append(row)
    return out


def set_wait_limit(iterations: int) -> int:
    """Iteration bound of the planner's two bounded waits for later plan
    calls in this process (negative: the default); returns the previous one.
    0 makes both waits take their fallback (MOONEP_ST_WAIT_TIMEOUT set, plan
    still exact)."""
    return _lib.moonep_set_wait_limit(int(iterations))


def set_cascade_capacity(capacity: int) -> int:
    """The replica capacity the relay cascade's guard compares with for later
    plan calls (<= 0: the plan's E + R - 1); returns the previous setting
    (0 for the default).  Lowering it makes the guard stricter; tests use it
    to put a repair step exactly on the limit."""
    return _lib.moonep_set_cascade_capacity(int(capacity))


def set_plan_path(mode: int) -> int:
    """Which planner later plan calls launch: 1 the two-kernel planner
    always, 0 (the default) the one-kernel planner where its CTAs all fit on
    the device at once; returns the previous setting.  Both give the same
    plan."""
    if mode not in (0, 1):
        raise ValueError(f"plan path must be 0 or 1, got {mode}")
    return _lib.moonep_set_plan_path(int(mode))


def abi_version() -> int:
    return _lib.moonep_abi_version()


def status_string(status: int) -> str:
    """Names of the MOONEP_ST_* bits set in a plan's status word ("ok" for 0)."""
    buf = ctypes.create_string_buffer(256)
    return _lib.moonep_status_string(int(status), buf, len(buf)).decode()
