"""The C ABI library loads, exports every symbol its header declares, and its
host-side checks agree with the oracle's configuration rules.  No GPU needed:
none of these calls launches a kernel."""
import re
import os

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moonep.h")).read()
    return re.findall(r"MOONEP_API\s+[\w\s\*]+?\b(moonep_\w+)\s*\(", src)


def test_header_declares_entry_points():
    names = _declared()
    for n in ("moonep_plan", "moonep_dispatch", "moonep_combine", "moonep_combine_backward",
              "moonep_reduce_replica_grads", "moonep_plan_sizes", "moonep_plan_layout"):
        assert n in names


def test_library_exports_every_declared_symbol(cuda_lib_path):
    import ctypes
    lib = ctypes.CDLL(cuda_lib_path)
    for n in _declared():
        assert hasattr(lib, n), n


def test_binding_loads(cuda_lib_path):
    from load_balancing_moonep_b200 import moonep
    assert moonep.abi_version() == 2
    for n in _declared():
        assert n in moonep.EXPORTED


def test_config_checks_match_oracle(cuda_lib_path):
    from load_balancing_moonep_b200 import moonep
    cases = [
        dict(R=4, E=16, K=2, S=8, H=8, B=2),
        dict(R=3, E=16, K=2, S=8, H=8, B=2),
        dict(R=4, E=16, K=2, S=8, H=8, B=3, flags=2),
        dict(R=4, E=16, K=2, S=8, H=8, B=4, flags=2),
        dict(R=4, E=16, K=2, S=8, H=8, B=13),
        dict(R=4, E=16, K=17, S=8, H=8, B=2),
        dict(R=0, E=16, K=2, S=8, H=8, B=2),
        dict(R=4, E=16, K=2, S=0, H=8, B=2),
        dict(R=32, E=384, K=8, S=4096, H=7168, B=12, flags=2),
        dict(R=64, E=384, K=8, S=128, H=7168, B=4),
    ]
    for c in cases:
        assert moonep.check_config(moonep.Config(**c)) == oracle.check_config(oracle.Config(**c)), c
    # flags: unknown bits are an argument error on both sides; the cascade
    # flag is known to both
    assert moonep.check_config(moonep.Config(R=4, E=16, K=2, S=8, H=8, B=2, flags=64)) == 1
    assert oracle.check_config(oracle.Config(R=4, E=16, K=2, S=8, H=8, B=2, flags=64)) == 1
    assert oracle.check_config(oracle.Config(R=4, E=16, K=2, S=8, H=8, B=2, flags=8)) == 0
    assert moonep.check_config(moonep.Config(R=4, E=16, K=2, S=8, H=8, B=2, flags=8)) == 0
    # the cascade's shared memory fits the large shape and E = R = 1024 with
    # the largest budget, and costs the plan nothing in device memory
    for c in (dict(R=32, E=384, K=8, S=4096, H=7168, B=12), dict(R=1024, E=1024, K=4, S=4, H=8, B=1023)):
        assert moonep.plan_sizes(moonep.Config(**c, flags=8)) == moonep.plan_sizes(moonep.Config(**c))
    # CUDA-only limits
    assert moonep.check_config(moonep.Config(R=4, E=16, K=2, S=8, H=12, B=2)) == 8
    assert moonep.check_config(moonep.Config(R=2, E=2048, K=2, S=8, H=8, B=2)) == 7
    with pytest.raises(moonep.MoonepError):
        moonep.plan_sizes(moonep.Config(R=3, E=16, K=2, S=8, H=8, B=2))


def test_plan_sizes_and_layout(cuda_lib_path):
    import ctypes
    from load_balancing_moonep_b200 import moonep
    cfg = moonep.Config(R=32, E=384, K=8, S=4096, H=7168, B=12)
    pb, wb = moonep.plan_sizes(cfg)
    n_pairs = cfg.pairs
    assert pb >= 4 * (2 * n_pairs + 384 + 3 * 32 * 385) and pb % 256 == 0
    assert wb >= 4 * 384 and wb % 256 == 0
    # layout of a fake, 256-aligned base address: host arithmetic only
    base = 1 << 40
    cp = moonep._CPlan()
    c = cfg.c()
    assert moonep._lib.moonep_plan_layout(ctypes.byref(c), base, ctypes.byref(cp)) == 0
    offs = [getattr(cp, f) - base for f in moonep.PLAN_FIELDS]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert offs[-1] < pb
    # misaligned base is rejected
    assert moonep._lib.moonep_plan_layout(ctypes.byref(c), base + 16, ctypes.byref(cp)) == 8


def test_status_string(cuda_lib_path):
    from load_balancing_moonep_b200 import moonep
    assert moonep.status_string(0) == "ok"
    assert moonep.status_string(moonep.ST_EXPERT_ID_RANGE) == "EXPERT_ID_RANGE"
    assert moonep.status_string(moonep.ST_OVERFLOW | moonep.ST_STRICT_VIOLATION) == "OVERFLOW|STRICT_VIOLATION"
    assert moonep.status_string(moonep.ST_WAIT_TIMEOUT | moonep.ST_WORKSPACE) == "WAIT_TIMEOUT|WORKSPACE"
    assert moonep.status_string(moonep.ST_ROW_RANGE | (1 << 7) | (1 << 12)) == "ROW_RANGE|bit7|bit12"
    import ctypes
    lib = ctypes.CDLL(cuda_lib_path)
    lib.moonep_status_string.restype = ctypes.c_char_p
    lib.moonep_status_string.argtypes = [ctypes.c_int, ctypes.c_char_p, ctypes.c_size_t]
    small = ctypes.create_string_buffer(6)
    assert lib.moonep_status_string(3, small, 6) == b"EXPER"  # truncated, NUL-terminated
    assert lib.moonep_status_string(3, None, 0) == b""


def test_single_gpu_planner_refuses_the_locality_flag(cuda_lib_path):
    """MOONEP_FLAG_LOCALITY is for expert parallelism (moonep_ep_plan): the
    one-GPU planner refuses it before touching memory."""
    import ctypes
    from load_balancing_moonep_b200 import moonep
    cfg = moonep.Config(R=4, E=16, K=2, S=8, H=8, B=2, flags=moonep.FLAG_LOCALITY)
    assert moonep.check_config(cfg) == 0
    cp = moonep._CPlan()
    for f in moonep.PLAN_FIELDS:  # non-null stand-ins: the call must not touch them
        setattr(cp, f, 1 << 20)
    c = cfg.c()
    assert moonep._lib.moonep_plan(ctypes.byref(c), 1 << 20, ctypes.byref(cp), 1 << 20, None) == 1
    assert moonep._lib.moonep_plan_noalloc(ctypes.byref(c), 1 << 20, ctypes.byref(cp), None) == 1


def test_host_setters_return_the_previous_setting(cuda_lib_path):
    """The three process-wide settings are host-only: each call returns the
    setting it replaces, and out-of-range values map as the header states
    (a negative wait bound restores the default 65536 iterations, a capacity
    <= 0 the plan's own E + R - 1 (reported as 0), any plan path other than 1
    the default 0).  The binding refuses plan paths other than 0 and 1."""
    import ctypes
    from load_balancing_moonep_b200 import moonep
    lib = ctypes.CDLL(cuda_lib_path)

    prev = moonep.set_wait_limit(5)
    try:
        assert moonep.set_wait_limit(-1) == 5
        assert moonep.set_wait_limit(0) == 65536
        assert moonep.set_wait_limit(7) == 0
        assert moonep.set_wait_limit(7) == 7
    finally:
        moonep.set_wait_limit(prev)

    prev = moonep.set_cascade_capacity(10)
    try:
        assert moonep.set_cascade_capacity(-3) == 10
        assert moonep.set_cascade_capacity(4) == 0
        assert moonep.set_cascade_capacity(0) == 4
        assert moonep.set_cascade_capacity(0) == 0
    finally:
        moonep.set_cascade_capacity(prev)

    prev = moonep.set_plan_path(1)
    try:
        assert lib.moonep_set_plan_path(5) == 1  # the C entry maps it to 0
        assert moonep.set_plan_path(0) == 0
        assert moonep.set_plan_path(1) == 0
        assert moonep.set_plan_path(1) == 1
        for bad in (2, -1):
            with pytest.raises(ValueError):
                moonep.set_plan_path(bad)
        assert moonep.set_plan_path(0) == 1  # the refused calls changed nothing
    finally:
        moonep.set_plan_path(prev)
