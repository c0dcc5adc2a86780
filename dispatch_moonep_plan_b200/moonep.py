"""Python binding of libmoonep.so (ctypes).  Argument marshalling only: every
step of the path runs in the library's CUDA kernels.  torch provides device
memory and streams.

The C ABI is declared in include/moonep.h; the names here match it:
``moonep_plan`` -> :func:`plan`, ``moonep_dispatch`` -> :func:`dispatch`, and
so on.  Importing this module fails loudly if the library has not been built;
there is no fallback.

Tensors are passed to the library as raw device addresses.  As in the C ABI,
each buffer must be a contiguous CUDA allocation of at least the byte count
:func:`sizes` gives for it: the library checks NULL pointers, alignment and
the configuration, but it cannot see a buffer's extent.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoonep.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_CUDA = 2
STATUS_OK = 0
STATUS_SLOT_BUDGET = 3
STATUS_BAD_INDEX = 4
STATUS_TIMEOUT = 5
STATUS_INTERNAL = 6
PAYLOAD_BF16 = 0
PAYLOAD_FP8 = 1
RULE_INDEX_ORDER = 0
RULE_KEEP_LIGHTEST = 1
RULE_LARGEST_FIRST = 2
EXPERT_IDENTITY = 0
EXPERT_SCALE = 1
MAX_E = 1024
MAX_R = 128
MAX_B = 64
MAX_K = 32
STATUS_WORDS = 8
NOALLOC_MAX_E = 512

# every symbol include/moonep.h declares
EXPORTS = ("moonep_version", "moonep_last_error", "moonep_sizes", "moonep_plan",
           "moonep_dispatch", "moonep_combine", "moonep_prefetch", "moonep_grad_reduce",
           "moonep_expert_standin", "moonep_plan_status", "moonep_weights_create",
           "moonep_weights_destroy", "moonep_set_wait_limit_ns",
           "moonep_debug_set_barrier_extra", "moonep_plan_noalloc", "moonep_combine_backward",
           "moonep_dispatch_backward", "moonep_expert_gemm")

i32, i64, sz, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p


class Config(ctypes.Structure):
    _fields_ = [("R", i32), ("S", i32), ("E", i32), ("K", i32), ("B", i32), ("H", i32),
                ("Hp", i32), ("payload", i32), ("rule", i32)]


class Sizes(ctypes.Structure):
    _fields_ = [("tokens", i64), ("picks", i64), ("rows_per_rank", i64),
                ("topk_idx_bytes", sz), ("topk_w_bytes", sz), ("x_bytes", sz),
                ("recv_bytes", sz), ("recv_scale_bytes", sz),
                ("dispatch_buffer_bytes_per_rank", sz), ("expert_out_bytes", sz),
                ("y_bytes", sz), ("expert_count_bytes", sz), ("rank_load_bytes", sz),
                ("slot_expert_bytes", sz), ("cu_seqlens_bytes", sz), ("dst_row_bytes", sz),
                ("src_of_row_bytes", sz), ("status_bytes", sz), ("maxvio_bytes", sz),
                ("workspace_bytes", sz), ("weight_row_bytes", sz),
                ("prefetch_pool_bytes_per_rank", sz), ("weights_view_bytes", sz)]


class Plan(ctypes.Structure):
    _fields_ = [("expert_count", vp), ("rank_load", vp), ("slot_expert", vp),
                ("cu_seqlens", vp), ("dst_row", vp), ("src_of_row", vp), ("status", vp),
                ("maxvio", vp), ("workspace", vp), ("workspace_bytes", sz)]


class Weights(ctypes.Structure):
    _fields_ = [("rank_view", vp * MAX_R), ("row_bytes", sz), ("view_bytes", sz),
                ("R", i32), ("E", i32), ("B", i32), ("elem_bytes", i32), ("impl", vp)]


class MoonEPError(RuntimeError):
    pass


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libmoonep.so is not built (%s); run "
                          "`python -m dispatch_moonep_plan_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    for name in EXPORTS:
        getattr(L, name)  # raises AttributeError if missing
    P = ctypes.POINTER
    L.moonep_version.restype = ctypes.c_int
    L.moonep_last_error.restype = ctypes.c_char_p
    L.moonep_sizes.argtypes = [P(Config), P(Sizes)]
    L.moonep_plan.argtypes = [P(Config), vp, P(Plan), vp]
    L.moonep_dispatch.argtypes = [P(Config), P(Plan), vp, vp, vp, vp]
    L.moonep_combine.argtypes = [P(Config), P(Plan), vp, vp, vp, vp]
    L.moonep_prefetch.argtypes = [P(Config), P(Plan), P(vp), i32, vp]
    L.moonep_grad_reduce.argtypes = [P(Config), P(Plan), P(vp), vp]
    L.moonep_expert_standin.argtypes = [P(Config), P(Plan), vp, vp, i32, vp, vp]
    L.moonep_plan_status.argtypes = [P(Plan), vp, P(i32)]
    L.moonep_weights_create.argtypes = [P(Config), i32, P(Weights)]
    L.moonep_weights_destroy.argtypes = [P(Weights)]
    L.moonep_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.moonep_debug_set_barrier_extra.argtypes = [i32]
    L.moonep_plan_noalloc.argtypes = [P(Config), vp, P(Plan), vp]
    L.moonep_combine_backward.argtypes = [P(Config), P(Plan), vp, vp, vp, vp, vp, vp]
    L.moonep_dispatch_backward.argtypes = [P(Config), P(Plan), vp, vp, vp]
    L.moonep_expert_gemm.argtypes = [P(Config), P(Plan), vp, vp, vp, vp, vp]
    return L


lib = _load()


def _check(rc, fn):
    if rc != OK:
        raise MoonEPError("%s failed (%d): %s" % (fn, rc, lib.moonep_last_error().decode()))


def config(R, S, E, K, B, H, Hp=0, payload=PAYLOAD_BF16, rule=RULE_INDEX_ORDER):
    return Config(R, S, E, K, B, H, Hp, payload, rule)


def config_from(d, rule=RULE_INDEX_ORDER):
    """Config from a workload dict (see workloads.WORKLOADS)."""
    payload = PAYLOAD_FP8 if d.get("payload") == "fp8" else PAYLOAD_BF16
    return Config(d["R"], d["S"], d["E"], d["K"], d["B"], d["H"], d.get("Hp", 0), payload, rule)


def sizes(cfg):
    out = Sizes()
    _check(lib.moonep_sizes(ctypes.byref(cfg), ctypes.byref(out)), "moonep_sizes")
    return out


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr() if hasattr(t, "data_ptr") else t)


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else stream)


class PlanBuffers:
    """Device buffers of one plan, allocated with torch, plus the C struct
    that points at them."""

    def __init__(self, cfg, device="cuda"):
        import torch
        s = sizes(cfg)
        T, K, R, E, B = s.tokens, cfg.K, cfg.R, cfg.E, cfg.B
        z = dict(dtype=torch.int32, device=device)
        self.cfg = cfg
        self.expert_count = torch.zeros(E, **z)
        self.rank_load = torch.zeros(R, **z)
        self.slot_expert = torch.zeros(max(R * B, 1), **z)
        self.cu_seqlens = torch.zeros(R * (E + B), **z)
        self.dst_row = torch.zeros(T * K, **z)
        self.src_of_row = torch.zeros(T * K, **z)
        self.status = torch.zeros(STATUS_WORDS, **z)
        self.maxvio = torch.zeros(1, dtype=torch.float64, device=device)
        self.workspace = torch.zeros(s.workspace_bytes // 4, **z)
        self.c = Plan(self.expert_count.data_ptr(), self.rank_load.data_ptr(),
                      self.slot_expert.data_ptr(), self.cu_seqlens.data_ptr(),
                      self.dst_row.data_ptr(), self.src_of_row.data_ptr(),
                      self.status.data_ptr(), self.maxvio.data_ptr(),
                      self.workspace.data_ptr(), s.workspace_bytes)

    def host(self):
        """Copy every plan output to host numpy arrays (synchronising)."""
        cfg = self.cfg
        T = cfg.R * cfg.S
        st = self.status.cpu().numpy()
        return dict(status=int(st[0]), fail_rank=int(st[1]), fail_slots=int(st[2]),
                    max_count=int(st[3]), maxvio=float(self.maxvio.item()),
                    expert_count=self.expert_count.cpu().numpy(),
                    rank_load=self.rank_load.cpu().numpy(),
                    slot_expert=self.slot_expert.cpu().numpy()[:cfg.R * cfg.B]
                    .reshape(cfg.R, cfg.B),
                    cu_seqlens=self.cu_seqlens.cpu().numpy().reshape(cfg.R, cfg.E + cfg.B),
                    dst_row=self.dst_row.cpu().numpy().reshape(T, cfg.K),
                    src_of_row=self.src_of_row.cpu().numpy())


def plan(cfg, topk_idx, bufs, stream=None):
    """moonep_plan: topk_idx int32 [T, K] device tensor (or pointer)."""
    _check(lib.moonep_plan(ctypes.byref(cfg), _ptr(topk_idx), ctypes.byref(bufs.c),
                           _stream(stream)), "moonep_plan")


def plan_noalloc(cfg, topk_idx, bufs, stream=None):
    """moonep_plan_noalloc: the planner without a caller workspace (the
    library's static scratch is used; ``bufs.c.workspace`` is ignored)."""
    _check(lib.moonep_plan_noalloc(ctypes.byref(cfg), _ptr(topk_idx), ctypes.byref(bufs.c),
                                   _stream(stream)), "moonep_plan_noalloc")


def dispatch(cfg, bufs, x, recv, recv_scale=None, stream=None):
    _check(lib.moonep_dispatch(ctypes.byref(cfg), ctypes.byref(bufs.c), _ptr(x), _ptr(recv),
                               _ptr(recv_scale), _stream(stream)), "moonep_dispatch")


def combine(cfg, bufs, expert_out, topk_w, y, stream=None):
    _check(lib.moonep_combine(ctypes.byref(cfg), ctypes.byref(bufs.c), _ptr(expert_out),
                              _ptr(topk_w), _ptr(y), _stream(stream)), "moonep_combine")


def combine_backward(cfg, bufs, dy, expert_out, topk_w, d_expert_out, d_topk_w, stream=None):
    _check(lib.moonep_combine_backward(ctypes.byref(cfg), ctypes.byref(bufs.c), _ptr(dy),
                                       _ptr(expert_out), _ptr(topk_w), _ptr(d_expert_out),
                                       _ptr(d_topk_w), _stream(stream)), "moonep_combine_backward")


def dispatch_backward(cfg, bufs, d_recv, dx, stream=None):
    _check(lib.moonep_dispatch_backward(ctypes.byref(cfg), ctypes.byref(bufs.c), _ptr(d_recv),
                                        _ptr(dx), _stream(stream)), "moonep_dispatch_backward")


def expert_standin(cfg, bufs, recv, recv_scale, mode, out, stream=None):
    _check(lib.moonep_expert_standin(ctypes.byref(cfg), ctypes.byref(bufs.c), _ptr(recv),
                                     _ptr(recv_scale), mode, _ptr(out), _stream(stream)),
           "moonep_expert_standin")


def expert_gemm(cfg, bufs, recv, weights, out, stream=None, recv_scale=None):
    """out[rows of group g of rank r] = recv[rows] @ weights[r][g]; ``weights``
    is the base of R consecutive [E+B, H, Hp] bf16 views (a tensor, a
    WeightViews' first view pointer, or an int address).  For the fp8
    payload, recv holds e4m3 codes and recv_scale their per-128 scales."""
    w = weights.data_ptr() if hasattr(weights, "data_ptr") else weights
    _check(lib.moonep_expert_gemm(ctypes.byref(cfg), ctypes.byref(bufs.c), _ptr(recv),
                                  _ptr(recv_scale), w, _ptr(out), _stream(stream)),
           "moonep_expert_gemm")


def _ptr_array(views):
    arr = (vp * len(views))()
    for i, v in enumerate(views):
        arr[i] = v.data_ptr() if hasattr(v, "data_ptr") else v
    return arr


def prefetch(cfg, bufs, rank_views, elem_bytes=2, stream=None):
    _check(lib.moonep_prefetch(ctypes.byref(cfg), ctypes.byref(bufs.c),
                               _ptr_array(rank_views), elem_bytes, _stream(stream)),
           "moonep_prefetch")


def grad_reduce(cfg, bufs, rank_views, stream=None):
    _check(lib.moonep_grad_reduce(ctypes.byref(cfg), ctypes.byref(bufs.c),
                                  _ptr_array(rank_views), _stream(stream)), "moonep_grad_reduce")


def plan_status(bufs, stream=None):
    out = (i32 * 4)()
    _check(lib.moonep_plan_status(ctypes.byref(bufs.c), _stream(stream), out),
           "moonep_plan_status")
    return list(out)


def set_wait_limit_ns(ns):
    _check(lib.moonep_set_wait_limit_ns(int(ns)), "moonep_set_wait_limit_ns")


def debug_set_barrier_extra(extra):
    _check(lib.moonep_debug_set_barrier_extra(int(extra)), "moonep_debug_set_barrier_extra")


class WeightViews:
    """R contiguous [E+B, H, Hp] views of one projection (moonep_weights_create);
    rows 0..E-1 of every view alias one physical home block."""

    def __init__(self, cfg, elem_bytes=2):
        self.w = Weights()
        _check(lib.moonep_weights_create(ctypes.byref(cfg), elem_bytes, ctypes.byref(self.w)),
               "moonep_weights_create")
        self.R = cfg.R
        self.ptrs = [self.w.rank_view[r] for r in range(cfg.R)]

    def close(self):
        if self.w.impl:
            _check(lib.moonep_weights_destroy(ctypes.byref(self.w)), "moonep_weights_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class _CudaArray:
    """Minimal __cuda_array_interface__ holder so torch can view foreign memory."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = dict(shape=tuple(shape), typestr=typestr,
                                             data=(int(ptr), False), version=3, strides=None)


def tensor_view(ptr, shape, dtype):
    """A torch tensor over device memory the library owns (no copy)."""
    import torch
    # __cuda_array_interface__ has no bfloat16: view such memory as int16
    carrier = torch.int16 if dtype == torch.bfloat16 else dtype
    typestr = {torch.int16: "<i2", torch.float16: "<f2", torch.float32: "<f4",
               torch.uint8: "|u1", torch.int32: "<i4"}[carrier]
    t = torch.as_tensor(_CudaArray(ptr, shape, typestr), device="cuda")
    return t.view(dtype) if carrier != dtype else t


def weight_view_tensor(views, r, cfg, dtype):
    """Rank r's [E+B, H, Hp] view of a WeightViews object as a torch tensor."""
    return tensor_view(views.ptrs[r], (cfg.E + cfg.B, cfg.H, cfg.Hp), dtype)
