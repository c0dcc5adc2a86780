"""The C-ABI library on a machine without a GPU: it builds, loads, exports
every entry point include/moonep.h declares, computes sizes, and rejects bad
arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moonep.h")


@pytest.fixture(scope="module")
def m():
    from dispatch_moonep_plan_b200 import build
    build.build()
    from dispatch_moonep_plan_b200 import moonep
    return moonep


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\w[\w\s\*]*?\b(moonep_\w+)\s*\(", text, re.M)))


def test_header_declares_what_binding_lists(m):
    assert _declared() == sorted(m.EXPORTS)


def test_library_exports_every_declared_symbol(m):
    out = subprocess.run(["nm", "-D", "--defined-only", m.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(moonep_\w+)$", out, re.M))
    for name in _declared():
        assert name in exported, name
        getattr(m.lib, name)


def test_version_and_sizes(m):
    assert m.lib.moonep_version() == 100
    cfg = m.config(16, 16384, 128, 8, 8, 4096, Hp=1536, payload=m.PAYLOAD_FP8)
    s = m.sizes(cfg)
    T, P, C = 16 * 16384, 16 * 16384 * 8, 16384 * 8
    assert (s.tokens, s.picks, s.rows_per_rank) == (T, P, C)
    assert s.recv_bytes == P * 4096 and s.recv_scale_bytes == P * 32 * 4
    assert s.dispatch_buffer_bytes_per_rank == C * 4096 + C * 32 * 4
    assert s.weight_row_bytes == 4096 * 1536 * 2
    assert s.prefetch_pool_bytes_per_rank == 8 * 4096 * 1536 * 2
    assert s.weights_view_bytes == 136 * 4096 * 1536 * 2
    assert s.cu_seqlens_bytes == 16 * 136 * 4 and s.slot_expert_bytes == 16 * 8 * 4
    assert s.status_bytes == m.STATUS_WORDS * 4


@pytest.mark.parametrize("bad,msg", [
    (dict(E=6, R=4), "multiple of R"),
    (dict(H=100), "multiple of 8"),
    (dict(payload=1, H=64), "128"),
    (dict(E=2048, R=2), "MAX_E"),
    (dict(R=256, E=256), "MAX_R"),
    (dict(B=65), "MAX_B"),
    (dict(K=33), "MAX_K"),
    (dict(S=1 << 28, K=8, R=1), "2\\^31"),
    (dict(S=0), "positive"),
    (dict(B=-1), "non-negative"),
    (dict(rule=3), "rule"),
])
def test_config_rejected(m, bad, msg):
    d = dict(R=2, S=8, E=4, K=2, B=2, H=64, Hp=0, payload=0, rule=0)
    d.update(bad)
    cfg = m.Config(**d)
    with pytest.raises(m.MoonEPError, match=msg):
        m.sizes(cfg)


def test_calls_reject_null_arguments_without_a_device(m):
    cfg = m.config(2, 8, 4, 2, 2, 64)
    plan = m.Plan()
    rc = m.lib.moonep_plan(ctypes.byref(cfg), None, ctypes.byref(plan), None)
    assert rc == m.ERR_INVALID_ARG and b"NULL" in m.lib.moonep_last_error()
    rc = m.lib.moonep_dispatch(ctypes.byref(cfg), ctypes.byref(plan), None, None, None, None)
    assert rc == m.ERR_INVALID_ARG
    rc = m.lib.moonep_combine(ctypes.byref(cfg), None, None, None, None, None)
    assert rc == m.ERR_INVALID_ARG
    rc = m.lib.moonep_plan_status(None, None, None)
    assert rc == m.ERR_INVALID_ARG
    rc = m.lib.moonep_weights_destroy(None)
    assert rc == m.ERR_INVALID_ARG
    assert m.lib.moonep_set_wait_limit_ns(0) == m.ERR_INVALID_ARG
    assert m.lib.moonep_debug_set_barrier_extra(-1) == m.ERR_INVALID_ARG


def test_workspace_checked_by_the_planner_only(m):
    """The planner rejects a missing workspace; calls that never read it
    (dispatch here) get past the plan checks without one and stop at their
    own first missing argument."""
    cfg = m.config(2, 8, 4, 2, 2, 64)
    fake = 16  # an aligned non-NULL address; nothing is launched
    plan = m.Plan(fake, fake, fake, fake, fake, fake, fake, fake, None, 0)
    rc = m.lib.moonep_plan(ctypes.byref(cfg), ctypes.c_void_p(fake), ctypes.byref(plan), None)
    assert rc == m.ERR_INVALID_ARG and b"workspace" in m.lib.moonep_last_error()
    rc = m.lib.moonep_dispatch(ctypes.byref(cfg), ctypes.byref(plan), None, None, None, None)
    assert rc == m.ERR_INVALID_ARG and b"x or recv is NULL" in m.lib.moonep_last_error()


def _fake_plan(m, slot=True):
    """A plan whose pointers are aligned non-NULL addresses; the calls below
    never get past their argument checks, so nothing reads them."""
    f = 16
    return m.Plan(f, f, f if slot else None, f, f, f, f, f, None, 0)


# (call, config overrides, arguments after (cfg, plan), expected message)
# Every case fails a check before any launch.
_F, _U = 16, 24  # aligned and 8-byte (not 16-byte) aligned fake addresses
_BAD_CALLS = [
    ("moonep_expert_gemm", dict(payload=1, H=128, Hp=128), (_F, None, _F, _F, None), "needs recv_scale"),
    ("moonep_expert_gemm", dict(payload=1, H=128, Hp=128), (_F, _U, _F, _F, None), "recv_scale must be 16-byte"),
    ("moonep_expert_gemm", dict(H=72, Hp=128), (_F, None, _F, _F, None), "multiple of 64"),
    ("moonep_expert_gemm", dict(Hp=0), (_F, None, _F, _F, None), "positive multiple of 128"),
    ("moonep_expert_gemm", dict(Hp=192), (_F, None, _F, _F, None), "positive multiple of 128"),
    ("moonep_expert_gemm", dict(Hp=128), (None, None, _F, _F, None), "NULL"),
    ("moonep_expert_gemm", dict(Hp=128), (_F, None, _U, _F, None), "16-byte aligned"),
    ("moonep_expert_standin", {}, (_F, None, 7, _F, None), "unknown mode"),
    ("moonep_expert_standin", dict(payload=1, H=128), (_F, None, 0, _F, None), "needs recv_scale"),
    ("moonep_expert_standin", {}, (_F, None, 0, _U, None), "16-byte aligned"),
    ("moonep_dispatch", {}, (_F, _F, _F, None), "takes no recv_scale"),
    ("moonep_dispatch", dict(payload=1, H=128), (_F, _F, None, None), "needs recv_scale"),
    ("moonep_dispatch", dict(payload=1, H=128), (_F, _F, _F + 2, None), "4-byte aligned"),
    ("moonep_dispatch", {}, (_U, _F, None, None), "16-byte aligned"),
    ("moonep_combine", {}, (_F, None, _F, None), "NULL"),
    ("moonep_combine", {}, (_F, _F, _U, None), "16-byte aligned"),
    ("moonep_combine_backward", {}, (_F, _F, _F, _F, None, None), "NULL argument"),
    ("moonep_combine_backward", {}, (_F, _U, _F, _F, _F, None), "16-byte aligned"),
    ("moonep_dispatch_backward", {}, (_F, None, None), "NULL"),
    ("moonep_dispatch_backward", {}, (_U, _F, None), "16-byte aligned"),
]


@pytest.mark.parametrize("fn,over,args,msg", _BAD_CALLS)
def test_calls_check_arguments_before_any_launch(m, fn, over, args, msg):
    d = dict(R=2, S=8, E=4, K=2, B=2, H=64, Hp=0, payload=0, rule=0)
    d.update(over)
    cfg = m.Config(**d)
    plan = _fake_plan(m)
    rc = getattr(m.lib, fn)(ctypes.byref(cfg), ctypes.byref(plan), *args)
    assert rc == m.ERR_INVALID_ARG
    assert msg in m.lib.moonep_last_error().decode(), m.lib.moonep_last_error()


def test_side_kernels_check_views_and_skip_without_slots(m):
    """prefetch and grad-reduce reject a missing or misaligned rank view and
    return OK without launching when the plan has no slots (B = 0)."""
    vp = ctypes.c_void_p
    views = (vp * 2)(16, 24)
    cfg = m.Config(2, 8, 4, 2, 2, 64, 128, 0, 0)
    plan = _fake_plan(m)
    assert m.lib.moonep_prefetch(ctypes.byref(cfg), ctypes.byref(plan), views, 2, None) == m.ERR_INVALID_ARG
    assert b"16-byte aligned" in m.lib.moonep_last_error()
    assert m.lib.moonep_prefetch(ctypes.byref(cfg), ctypes.byref(plan), views, 3, None) == m.ERR_INVALID_ARG
    assert b"elem_bytes" in m.lib.moonep_last_error()
    assert m.lib.moonep_grad_reduce(ctypes.byref(cfg), ctypes.byref(plan), None, None) == m.ERR_INVALID_ARG
    assert b"rank_grads is NULL" in m.lib.moonep_last_error()
    cfg0 = m.Config(2, 8, 4, 2, 0, 64, 128, 0, 0)
    plan0 = _fake_plan(m, slot=False)
    ok_views = (vp * 2)(16, 32)
    assert m.lib.moonep_prefetch(ctypes.byref(cfg0), ctypes.byref(plan0), ok_views, 2, None) == m.OK
    assert m.lib.moonep_grad_reduce(ctypes.byref(cfg0), ctypes.byref(plan0), ok_views, None) == m.OK
    # a plan with slots needs slot_expert
    rc = m.lib.moonep_prefetch(ctypes.byref(cfg), ctypes.byref(_fake_plan(m, slot=False)), ok_views, 2, None)
    assert rc == m.ERR_INVALID_ARG and b"slot_expert" in m.lib.moonep_last_error()
