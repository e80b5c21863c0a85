"""ctypes binding of libprism (include/prism.h): argument marshalling only.

Every step of the plan and of the attention runs in the library's CUDA
kernels; this module passes device pointers, sizes and the current CUDA stream
through, allocates outputs with torch, and raises on a non-zero status.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libprism.so")

PRISM_OK = 0
PRISM_ERR_INVALID_ARG = 1
PRISM_ERR_WORKSPACE = 2
PRISM_ERR_CUDA = 3
PRISM_ERR_TIMEOUT = 4
PRISM_ERR_DEVICE_CHECK = 5
PRISM_ERR_UNSUPPORTED = 6
PRISM_ERR_SCRATCH_LIMIT = 7

PRISM_BF16 = 0
PRISM_F32 = 1

ITEMS = {
    "shape_id": (0, np.uint8), "nblocks": (1, np.int32), "blk_start": (2, np.int32),
    "sel_bits": (3, np.uint32), "row_ptr": (4, np.int32), "col_idx": (5, np.int32),
    "col_ptr": (6, np.int32), "row_idx": (7, np.int32), "qbar": (8, np.float32),
    "kbar": (9, np.float32), "src": (10, np.int32), "zone_stats": (11, np.float32),
    "zone_cut": (12, np.uint8), "shape_id2": (13, np.uint8), "zone_energy": (14, np.float32),
    "region_stats": (15, np.float32), "list_offsets": (16, np.int64), "qkv_max": (17, np.uint32),
}


PRISM_SHAPE_DYNAMIC = 0
PRISM_SHAPE_ISOTROPIC = 1
PRISM_SHAPE_FIXED = 2


class PrismParams(C.Structure):
    _fields_ = [("T", C.c_int32), ("H", C.c_int32), ("W", C.c_int32), ("heads", C.c_int32),
                ("head_dim", C.c_int32), ("dtype", C.c_int32), ("out_dtype", C.c_int32),
                ("top_k", C.c_int32),
                ("top_p", C.c_float), ("eps", C.c_float), ("tau128", C.c_float),
                ("tau256", C.c_float), ("alpha", C.c_float), ("shape_mode", C.c_int32),
                ("fixed_shape", C.c_int32), ("top_k_frac", C.c_float), ("cut_ratio", C.c_float)]


class PrismError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def load(path: str | None = None) -> C.CDLL:
    """Load libprism.so; raises if it is missing (there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or os.environ.get("PRISM_LIB") or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libprism.so not built at {p}: run "
                          "`python -m dynamic_block_sparse_indicator_b200.build`")
    lib = C.CDLL(p)
    vp, i32, sz = C.c_void_p, C.c_int, C.c_size_t
    pp = C.POINTER(PrismParams)
    sig = {
        "prism_plan_workspace_bytes": (sz, [pp]),
        "prism_plan_core_bytes": (sz, [pp]),
        "prism_plan_list_bytes": (i32, [vp, C.POINTER(sz), vp]),
        "prism_plan_attach_lists": (i32, [vp, vp, sz, vp]),
        "prism_plan": (i32, [pp, vp, vp, vp, vp, vp, sz, vp, C.POINTER(vp)]),
        "prism_plan_sharded": (i32, [pp, C.POINTER(vp), C.POINTER(vp), C.POINTER(vp), i32, i32, i32, vp,
                                     vp, sz, vp, C.POINTER(vp)]),
        "prism_plan_import_sharded": (i32, [pp, C.POINTER(vp), C.POINTER(vp), C.POINTER(vp), i32, i32, i32, vp,
                                            vp, vp, vp, vp, sz, vp, C.POINTER(vp)]),
        "prism_plan_import": (i32, [pp, vp, vp, vp, vp, vp, vp, sz, vp, C.POINTER(vp)]),
        "prism_plan_import_cuts": (i32, [pp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, C.POINTER(vp)]),
        "prism_attn_fwd": (i32, [vp, vp, vp, vp]),
        "prism_attn_fwd_sharded": (i32, [vp, C.POINTER(vp), i32, i32, i32, vp, vp]),
        "prism_attn_bwd_sharded": (i32, [vp, C.POINTER(vp), C.POINTER(vp), vp, C.POINTER(vp), C.POINTER(vp),
                                         C.POINTER(vp), i32, i32, i32, vp]),
        "prism_attn_bwd": (i32, [vp, vp, vp, vp, vp, vp, vp, vp]),
        "prism_plan_item_bytes": (sz, [vp, i32]),
        "prism_plan_export": (i32, [vp, i32, vp, sz, vp]),
        "prism_get_status": (i32, [vp, vp]),
        "prism_get_status_ex": (i32, [vp, C.POINTER(C.c_int32), vp]),
        "prism_selftest_timeout": (i32, [vp, vp]),
        "prism_plan_destroy": (None, [vp]),
        "prism_status_string": (C.c_char_p, [i32]),
        "prism_version": (C.c_char_p, []),
        "prism_profile_enable": (i32, [vp, i32]),
        "prism_profile_plans": (i32, [i32]),
        "prism_profile_read": (i32, [vp, C.POINTER(C.c_float), C.POINTER(C.c_int), vp]),
        "prism_launch_count": (C.c_int64, [vp]),
        "prism_zone_shapes_noalloc": (i32, [pp, vp, vp, vp, vp, vp]),
        "prism_av_norm": (i32, [C.c_int64, C.c_int32, C.c_int32, C.c_int32, vp, vp, vp, vp, vp,
                                C.c_int32, vp, vp]),
        "prism_status_read": (i32, [vp, C.POINTER(C.c_int32), vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def profile_plans(on: bool = True) -> bool:
    """Plans created afterwards time their own plan kernels (process-wide); returns the old setting."""
    return bool(load().prism_profile_plans(1 if on else 0))


def status_string(st: int) -> str:
    return load().prism_status_string(st).decode()


def make_params(T, H, W, heads, head_dim, dtype, top_k, top_p, eps, tau128=0.5, tau256=0.25,
                out_dtype=PRISM_F32, alpha=0.5, shape_mode=PRISM_SHAPE_DYNAMIC, fixed_shape=0,
                top_k_frac=0.0, cut_ratio=0.0):
    return PrismParams(T, H, W, heads, head_dim, dtype, out_dtype, top_k, float(top_p),
                       float(eps), float(tau128), float(tau256), float(alpha), int(shape_mode),
                       int(fixed_shape), float(top_k_frac), float(cut_ratio))


def workspace_bytes(params: PrismParams) -> int:
    """Workspace of a plan ready in one call (index lists at their dense bound)."""
    return int(load().prism_plan_workspace_bytes(C.byref(params)))


def core_bytes(params: PrismParams) -> int:
    """Workspace without the index lists (they go to a second buffer sized after planning)."""
    return int(load().prism_plan_core_bytes(C.byref(params)))


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _addresses(xs):
    """A ctypes array of device addresses from tensors or ints."""
    return (C.c_void_p * len(xs))(*[x if isinstance(x, int) else x.data_ptr() for x in xs])


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


class Plan:
    """A plan handle plus the device buffers it points into (kept alive here)."""

    def __init__(self, params, handle, workspace, inputs, lists=None):
        self.params = params
        self._h = handle
        self._ws = workspace
        self._lists = lists            # the index lists' buffer of a two-call plan
        self._inputs = inputs          # Q, K, V must outlive the plan

    @property
    def handle(self):
        return self._h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:
            _lib.prism_plan_destroy(h)
            self._h = None

    @property
    def N(self):
        p = self.params
        return p.T * p.H * p.W

    def _out_dtype(self):
        import torch
        return torch.float32 if self.params.out_dtype == PRISM_F32 else torch.bfloat16

    def attn_fwd(self, O=None, lse=None, stream=None):
        import torch
        p = self.params
        dev = self._ws.device
        if O is None:
            O = torch.empty(p.heads, self.N, p.head_dim, dtype=self._out_dtype(), device=dev)
        if lse is None:
            lse = torch.empty(p.heads, self.N, dtype=torch.float32, device=dev)
        st = load().prism_attn_fwd(self._h, _ptr(O), _ptr(lse), _stream(stream))
        if st:
            raise PrismError(st, "prism_attn_fwd")
        return O, lse

    def attn_bwd(self, dO, O, lse, dQ=None, dK=None, dV=None, stream=None):
        import torch
        p = self.params
        dev = self._ws.device
        mk = lambda: torch.empty(p.heads, self.N, p.head_dim, dtype=self._out_dtype(), device=dev)
        dQ = mk() if dQ is None else dQ
        dK = mk() if dK is None else dK
        dV = mk() if dV is None else dV
        st = load().prism_attn_bwd(self._h, _ptr(dO), _ptr(O), _ptr(lse), _ptr(dQ), _ptr(dK),
                                   _ptr(dV), _stream(stream))
        if st:
            raise PrismError(st, "prism_attn_bwd")
        return dQ, dK, dV

    def attn_fwd_sharded(self, O_shards, head0, heads_total, lse=None, stream=None):
        """The forward writing O into token shards (lists of [heads_total, N/n, D] tensors or
        device addresses, shard s = frames [s T/n, (s + 1) T/n)): rows of this plan's heads
        head0 .. head0 + heads - 1.  The LSE stays [heads, N] on this device."""
        import torch
        p = self.params
        if lse is None:
            lse = torch.empty(p.heads, self.N, dtype=torch.float32, device=self._ws.device)
        arr = _addresses(O_shards)
        st = load().prism_attn_fwd_sharded(self._h, arr, len(O_shards), int(heads_total), int(head0), _ptr(lse),
                                           _stream(stream))
        if st:
            raise PrismError(st, "prism_attn_fwd_sharded")
        return lse

    def attn_bwd_sharded(self, dO_shards, O_shards, lse, dQ_shards, dK_shards, dV_shards, head0, heads_total,
                         stream=None):
        """The backward reading dO and O from token shards and writing dQ, dK, dV into token
        shards (the layout of attn_fwd_sharded)."""
        n = len(dO_shards)
        if not all(len(x) == n for x in (O_shards, dQ_shards, dK_shards, dV_shards)):
            raise ValueError("every shard list must have the same length")
        st = load().prism_attn_bwd_sharded(self._h, _addresses(dO_shards), _addresses(O_shards), _ptr(lse),
                                           _addresses(dQ_shards), _addresses(dK_shards), _addresses(dV_shards),
                                           n, int(heads_total), int(head0), _stream(stream))
        if st:
            raise PrismError(st, "prism_attn_bwd_sharded")

    def export(self, item: str, stream=None) -> np.ndarray:
        code, dt = ITEMS[item]
        lib = load()
        nbytes = int(lib.prism_plan_item_bytes(self._h, code))
        out = np.empty(nbytes // np.dtype(dt).itemsize, dtype=dt)
        st = lib.prism_plan_export(self._h, code, out.ctypes.data_as(C.c_void_p), nbytes,
                                   _stream(stream))
        if st:
            raise PrismError(st, f"prism_plan_export({item})")
        return out

    STAGES = ("fwd", "bwd_pre", "bwd_dkdv", "bwd_dq", "plan_stats", "plan_shapes", "plan_gather",
              "plan_select", "plan_lists")

    def profile(self, on: bool = True):
        load().prism_profile_enable(self._h, 1 if on else 0)

    def profile_read(self, stream=None):
        """{stage: (ms, launches)} accumulated since the last read (synchronises)."""
        ms = (C.c_float * len(self.STAGES))()
        n = (C.c_int * len(self.STAGES))()
        st = load().prism_profile_read(self._h, ms, n, _stream(stream))
        if st:
            raise PrismError(st, "prism_profile_read")
        return {k: (float(ms[i]), int(n[i])) for i, k in enumerate(self.STAGES)}

    def launches(self) -> int:
        return int(load().prism_launch_count(self._h))

    def status(self, stream=None) -> int:
        return int(load().prism_get_status(self._h, _stream(stream)))

    def status_ex(self, stream=None):
        """(status, site of a timed-out wait) -- synchronises and clears."""
        site = C.c_int32(0)
        st = load().prism_get_status_ex(self._h, C.byref(site), _stream(stream))
        return int(st), int(site.value)

    def selftest_timeout(self, stream=None):
        st = load().prism_selftest_timeout(self._h, _stream(stream))
        if st:
            raise PrismError(st, "prism_selftest_timeout")


def _check_inputs(Q, K, V, params):
    import torch
    want = torch.float32 if params.dtype == PRISM_F32 else torch.bfloat16
    N = params.T * params.H * params.W
    for t in (Q, K, V):
        if t.dtype != want or not t.is_cuda or not t.is_contiguous():
            raise ValueError("Q, K, V must be contiguous CUDA tensors of the plan's dtype")
        if tuple(t.shape) != (params.heads, N, params.head_dim):
            raise ValueError(f"expected [heads, N, D] = {(params.heads, N, params.head_dim)}, "
                             f"got {tuple(t.shape)}")


def _attach_lists(lib, h, device, stream):
    """Size and build a two-call plan's index lists in a buffer of their own."""
    import torch
    nbytes = C.c_size_t(0)
    st = lib.prism_plan_list_bytes(h, C.byref(nbytes), _stream(stream))
    if st:
        raise PrismError(st, "prism_plan_list_bytes")
    lists = torch.empty(max(int(nbytes.value), 16), dtype=torch.uint8, device=device)
    st = lib.prism_plan_attach_lists(h, _ptr(lists), lists.numel(), _stream(stream))
    if st:
        raise PrismError(st, "prism_plan_attach_lists")
    return lists


def plan(Q, K, V, a_map, params: PrismParams, workspace=None, stream=None, compact=False) -> Plan:
    """Stages 1-3 on the GPU.  Q, K, V: [heads, N, D] CUDA tensors (raster order).
    compact=True plans with the core workspace and sizes the index lists from
    their counts (one stream synchronisation) instead of their dense bound."""
    import torch
    lib = load()
    _check_inputs(Q, K, V, params)
    need = core_bytes(params) if compact else workspace_bytes(params)
    if need == 0:
        raise PrismError(PRISM_ERR_INVALID_ARG, "prism_plan_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    h = C.c_void_p()
    st = lib.prism_plan(C.byref(params), _ptr(Q), _ptr(K), _ptr(V), _ptr(a_map), _ptr(workspace),
                        workspace.numel(), _stream(stream), C.byref(h))
    if st:
        raise PrismError(st, "prism_plan")
    lists = None
    if workspace.numel() < workspace_bytes(params):
        try:
            lists = _attach_lists(lib, h, Q.device, stream)
        except PrismError:
            lib.prism_plan_destroy(h)
            raise
    return Plan(params, h, workspace, (Q, K, V, a_map), lists)


def _shard_args(Qs, Ks, Vs, params, heads_total):
    """Checks a shard layout; returns (address arrays, heads_total, device, tensors)."""
    import torch
    n = len(Qs)
    if n == 0 or len(Ks) != n or len(Vs) != n:
        raise ValueError("Qs, Ks, Vs must be non-empty lists of the same length")
    N = params.T * params.H * params.W
    if params.T % n:
        raise ValueError(f"{n} shards do not divide T = {params.T}")
    want = torch.float32 if params.dtype == PRISM_F32 else torch.bfloat16
    device, tensors = None, []
    for t in (*Qs, *Ks, *Vs):
        if isinstance(t, int):
            continue
        if t.dtype != want or not t.is_cuda or not t.is_contiguous():
            raise ValueError("shards must be contiguous CUDA tensors of the plan's dtype (or device addresses)")
        if heads_total is None:
            heads_total = t.shape[0]
        if tuple(t.shape) != (heads_total, N // n, params.head_dim):
            raise ValueError(f"expected shards of [heads_total, N/shards, D] = "
                             f"{(heads_total, N // n, params.head_dim)}, got {tuple(t.shape)}")
        device = device or t.device
        tensors.append(t)
    if heads_total is None:
        raise ValueError("heads_total is needed when every shard is given as an address")
    device = device or torch.device("cuda", torch.cuda.current_device())
    return [_addresses(xs) for xs in (Qs, Ks, Vs)], int(heads_total), device, tuple(tensors)


def plan_import_sharded(Qs, Ks, Vs, shape_id, sel_bits, params: PrismParams, head0=0, heads_total=None,
                        zone_cut=None, shape_id2=None, workspace=None, stream=None, compact=False) -> Plan:
    """plan_import for inputs held as token shards (the layout of plan_sharded)."""
    import torch
    lib = load()
    arrs, heads_total, device, tensors = _shard_args(Qs, Ks, Vs, params, heads_total)
    need = core_bytes(params) if compact else workspace_bytes(params)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    h = C.c_void_p()
    st = lib.prism_plan_import_sharded(C.byref(params), arrs[0], arrs[1], arrs[2], len(Qs), heads_total,
                                       int(head0), _ptr(shape_id), _ptr(zone_cut), _ptr(shape_id2),
                                       _ptr(sel_bits), _ptr(workspace), workspace.numel(), _stream(stream),
                                       C.byref(h))
    if st:
        raise PrismError(st, "prism_plan_import_sharded")
    lists = None
    if workspace.numel() < workspace_bytes(params):
        try:
            lists = _attach_lists(lib, h, device, stream)
        except PrismError:
            lib.prism_plan_destroy(h)
            raise
    return Plan(params, h, workspace, (tensors, shape_id, sel_bits, zone_cut, shape_id2), lists)


def plan_sharded(Qs, Ks, Vs, a_map, params: PrismParams, head0=0, heads_total=None, workspace=None,
                 stream=None, compact=False) -> Plan:
    """Stages 1-3 for heads head0 .. head0 + params.heads - 1 of inputs held as
    token shards: Qs, Ks, Vs are equal-length lists (one entry per shard, shard s
    holding frames [s T/n, (s + 1) T/n) of every head as [heads_total, N/n, D]),
    each a contiguous CUDA tensor or a raw device address (an int: another GPU's
    shard mapped for peer access).  The plan then runs like `plan` on those heads."""
    import torch
    lib = load()
    arrs, heads_total, device, tensors = _shard_args(Qs, Ks, Vs, params, heads_total)
    n = len(Qs)
    need = core_bytes(params) if compact else workspace_bytes(params)
    if need == 0:
        raise PrismError(PRISM_ERR_INVALID_ARG, "prism_plan_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    h = C.c_void_p()
    st = lib.prism_plan_sharded(C.byref(params), arrs[0], arrs[1], arrs[2], n, int(heads_total), int(head0),
                                _ptr(a_map), _ptr(workspace), workspace.numel(), _stream(stream), C.byref(h))
    if st:
        raise PrismError(st, "prism_plan_sharded")
    lists = None
    if workspace.numel() < workspace_bytes(params):
        try:
            lists = _attach_lists(lib, h, device, stream)
        except PrismError:
            lib.prism_plan_destroy(h)
            raise
    return Plan(params, h, workspace, (tensors, a_map), lists)


def plan_import(Q, K, V, shape_id, sel_bits, params: PrismParams, workspace=None, stream=None,
                zone_cut=None, shape_id2=None, compact=False) -> Plan:
    """A plan from given shape ids [heads, Nz] (uint8) and selection bitmap (int32/uint32 words);
    with adaptive temporal boundaries also the split frames zone_cut and the second parts'
    shapes shape_id2 ([heads, Nz] uint8 each)."""
    import torch
    lib = load()
    _check_inputs(Q, K, V, params)
    need = core_bytes(params) if compact else workspace_bytes(params)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    h = C.c_void_p()
    if zone_cut is None:
        st = lib.prism_plan_import(C.byref(params), _ptr(Q), _ptr(K), _ptr(V), _ptr(shape_id),
                                   _ptr(sel_bits), _ptr(workspace), workspace.numel(), _stream(stream),
                                   C.byref(h))
    else:
        st = lib.prism_plan_import_cuts(C.byref(params), _ptr(Q), _ptr(K), _ptr(V), _ptr(shape_id),
                                        _ptr(zone_cut), _ptr(shape_id2), _ptr(sel_bits), _ptr(workspace),
                                        workspace.numel(), _stream(stream), C.byref(h))
    if st:
        raise PrismError(st, "prism_plan_import")
    lists = None
    if workspace.numel() < workspace_bytes(params):
        try:
            lists = _attach_lists(lib, h, Q.device, stream)
        except PrismError:
            lib.prism_plan_destroy(h)
            raise
    return Plan(params, h, workspace, (Q, K, V, shape_id, sel_bits, zone_cut, shape_id2), lists)


def av_norm(Qv, Ka, Va, a_map=None, h_hat=None, hhat_dtype=None, want_hhat=False, status=None,
            stream=None):
    """The guidance map a [N] (fp32) = || CrossAttn(Qv, Ka, Va) ||_2 over the heads, and
    optionally h_hat [heads, N, D].  Qv [heads, N, D], Ka, Va [heads, M, D]: contiguous
    bf16 CUDA tensors.  `status` is a device int32[4] block (zeroed here when created);
    read it with status_read()."""
    import torch
    for t in (Qv, Ka, Va):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError("Qv, Ka, Va must be contiguous 3-D bf16 CUDA tensors")
    heads, N, D = Qv.shape
    M = Ka.shape[1]
    if tuple(Ka.shape) != (heads, M, D) or tuple(Va.shape) != (heads, M, D):
        raise ValueError(f"Ka, Va must be [heads, M, D] = [{heads}, M, {D}]")
    dev = Qv.device
    if a_map is None:
        a_map = torch.empty(N, dtype=torch.float32, device=dev)
    if hhat_dtype is None:
        hhat_dtype = PRISM_BF16 if h_hat is None or h_hat.dtype == torch.bfloat16 else PRISM_F32
    if h_hat is None and want_hhat:
        dt = torch.float32 if hhat_dtype == PRISM_F32 else torch.bfloat16
        h_hat = torch.empty(heads, N, D, dtype=dt, device=dev)
    if status is None:
        status = torch.zeros(4, dtype=torch.int32, device=dev)
    st = load().prism_av_norm(int(N), int(M), int(heads), int(D), _ptr(Qv), _ptr(Ka), _ptr(Va),
                              _ptr(a_map), _ptr(h_hat), int(hhat_dtype), _ptr(status),
                              _stream(stream))
    if st:
        raise PrismError(st, "prism_av_norm")
    return a_map, h_hat, status


def status_read(status, stream=None):
    """(status, site) of a device status block; synchronises and clears it."""
    site = C.c_int32(0)
    st = load().prism_status_read(_ptr(status), C.byref(site), _stream(stream))
    return int(st), int(site.value)
