"""B200-native ZeRO partitioned mixed-precision Adam step.

Thin Python binding of ``libzero.so`` (C ABI in ``include/zero.h``): the same
entry points, with torch tensors turned into device pointers and the current
torch stream passed as the CUDA stream.  Every step of the computation runs
in the library's sm_100a kernels; there is no Python or CPU fallback -- if the
library is missing, every call raises.

    plan = zero_plan(psi, nd, stage, bucket_elems, unit_elems=[...])
    zero_step(plan, grads, master, exp_avg, exp_avg_sq, params, adam, t)
    zero_gather_layer(plan, u, owner_params, full_layer)   # stage 3
    zero_release_layer(plan, u)
"""
import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libzero.so")

# status codes (zero_status_t)
ZERO_OK, ZERO_EINVAL, ZERO_ENOMEM, ZERO_ECUDA, ZERO_ESTATE, ZERO_ETIMEOUT = range(6)

# queries (zero_query_t)
(ZERO_Q_PSI, ZERO_Q_PSI_PAD, ZERO_Q_S, ZERO_Q_ND, ZERO_Q_STAGE, ZERO_Q_N_UNITS,
 ZERO_Q_UNIT_LEN, ZERO_Q_UNIT_PAD, ZERO_Q_UNIT_SHARD, ZERO_Q_UNIT_BASE,
 ZERO_Q_UNIT_OFFSET, ZERO_Q_N_BUCKETS, ZERO_Q_BUCKET_UNIT, ZERO_Q_BUCKET_BEGIN,
 ZERO_Q_BUCKET_END, ZERO_Q_OWNER, ZERO_Q_OWNER_OFFSET, ZERO_Q_MEM_BYTES_PER_RANK,
 ZERO_Q_WORKSPACE_BYTES, ZERO_Q_LIVE_UNITS, ZERO_Q_PEAK_LIVE_UNITS,
 ZERO_Q_PEAK_LIVE_BYTES, ZERO_Q_IS_LIVE, ZERO_Q_MAX_LIVE, ZERO_Q_ALIGN,
 ZERO_Q_BUCKET_ELEMS, ZERO_Q_STATE_REPLICAS, ZERO_Q_GRAD_REPLICAS, ZERO_Q_PARAM_REPLICAS,
 ZERO_Q_LOST_RANK_UNRECOVERABLE) = range(30)

# accounting kinds (zero_bytes_kind_t) and flags
(ZERO_BYTES_COMM_ELEMS_PER_RANK, ZERO_BYTES_COMM_PER_RANK, ZERO_BYTES_HBM_STEP,
 ZERO_BYTES_HBM_GATHER_STEP, ZERO_BYTES_HBM_GUARDED_STEP) = range(5)
ZERO_BYTES_FLAG_OWNER_VIEW = 1
ZERO_BYTES_FLAG_REDUCED = 2


class ZeroError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("%s (%s)" % (message, status))
        self.status = status


class _PlanDesc(ctypes.Structure):
    _fields_ = [("psi", ctypes.c_uint64), ("nd", ctypes.c_uint32),
                ("stage", ctypes.c_uint32), ("bucket_elems", ctypes.c_uint64),
                ("align_elems", ctypes.c_uint32), ("k_bytes", ctypes.c_uint32),
                ("n_units", ctypes.c_uint32), ("max_live", ctypes.c_uint32),
                ("unit_elems", ctypes.POINTER(ctypes.c_uint64))]


class _Adam(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double),
                ("beta2", ctypes.c_double), ("eps", ctypes.c_double),
                ("grad_scale", ctypes.c_double), ("weight_decay", ctypes.c_double)]


class _Guard(ctypes.Structure):
    _fields_ = [("max_grad_norm", ctypes.c_double), ("skip_nonfinite", ctypes.c_int32)]


class _Bufs(ctypes.Structure):
    _fields_ = [("grads", ctypes.c_void_p), ("grad_stride", ctypes.c_uint64),
                ("master", ctypes.c_void_p), ("exp_avg", ctypes.c_void_p),
                ("exp_avg_sq", ctypes.c_void_p), ("params", ctypes.c_void_p),
                ("param_stride", ctypes.c_uint64), ("reduced_grad", ctypes.c_void_p),
                ("grad_norm_sq", ctypes.c_void_p), ("overflow", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_uint64),
                ("owner_view", ctypes.c_int32), ("adam_consts", ctypes.c_void_p)]


class _PeerBufs(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_uint32), ("reserved", ctypes.c_uint32),
                ("grads", ctypes.POINTER(ctypes.c_void_p)), ("params", ctypes.POINTER(ctypes.c_void_p)),
                ("master", ctypes.c_void_p), ("exp_avg", ctypes.c_void_p),
                ("exp_avg_sq", ctypes.c_void_p), ("reduced_grad", ctypes.c_void_p),
                ("grad_norm_sq", ctypes.c_void_p), ("overflow", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_uint64),
                ("adam_consts", ctypes.c_void_p)]


class _IpcHandle(ctypes.Structure):
    _fields_ = [("handle", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64),
                ("alloc_bytes", ctypes.c_uint64), ("exporter_va", ctypes.c_uint64),
                ("device", ctypes.c_int32), ("exporter_pid", ctypes.c_int32)]


ZERO_MAX_PEERS = 128
IPC_HANDLE_BYTES = ctypes.sizeof(_IpcHandle)

_LIB = None


def lib():
    """The loaded libzero.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libzero.so is missing (%s); build it with "
                "`python -m zero_partitioned_optimizer_step_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        st = ctypes.c_int
        vp = ctypes.c_void_p
        u64 = ctypes.c_uint64
        L.zero_plan.restype = st
        L.zero_plan.argtypes = [ctypes.POINTER(_PlanDesc), ctypes.POINTER(vp)]
        L.zero_plan_destroy.restype = None
        L.zero_plan_destroy.argtypes = [vp]
        L.zero_plan_query.restype = st
        L.zero_plan_query.argtypes = [vp, ctypes.c_int, u64, ctypes.POINTER(u64)]
        L.zero_step.restype = st
        L.zero_step.argtypes = [vp, ctypes.POINTER(_Bufs), ctypes.POINTER(_Adam), u64, vp]
        L.zero_step_noalloc.restype = st
        L.zero_step_noalloc.argtypes = [vp, ctypes.POINTER(_Bufs), ctypes.POINTER(_Adam), u64, vp]
        L.zero_step_guarded.restype = st
        L.zero_step_guarded.argtypes = [vp, ctypes.POINTER(_Bufs), ctypes.POINTER(_Adam),
                                        ctypes.POINTER(_Guard), u64, vp]
        L.zero_step_buckets.restype = st
        L.zero_step_buckets.argtypes = [vp, ctypes.POINTER(_Bufs), ctypes.POINTER(_Adam),
                                        u64, u64, u64, vp]
        L.zero_gather_layer.restype = st
        L.zero_gather_layer.argtypes = [vp, ctypes.c_uint32, vp, vp, vp]
        L.zero_release_layer.restype = st
        L.zero_release_layer.argtypes = [vp, ctypes.c_uint32]
        L.zero_bytes_moved.restype = st
        L.zero_bytes_moved.argtypes = [vp, ctypes.c_int, ctypes.c_uint32, ctypes.POINTER(u64)]
        L.zero_step_kernel.restype = st
        L.zero_step_kernel.argtypes = [vp, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint32)]
        L.zero_step_peers_kernel.restype = st
        L.zero_step_peers_kernel.argtypes = [vp, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_uint64,
                                             ctypes.POINTER(ctypes.c_uint32)]
        L.zero_reshard.restype = st
        L.zero_reshard.argtypes = [vp, vp, vp, vp, ctypes.c_uint32, vp]
        L.zero_adam_consts.restype = st
        L.zero_adam_consts.argtypes = [ctypes.POINTER(_Adam), u64, vp]
        L.zero_stream_status.restype = st
        L.zero_stream_status.argtypes = [vp]
        L.zero_step_peers.restype = st
        L.zero_step_peers.argtypes = [vp, ctypes.POINTER(_PeerBufs), ctypes.POINTER(_Adam),
                                      u64, u64, u64, vp]
        L.zero_gather_layer_peers.restype = st
        L.zero_gather_layer_peers.argtypes = [vp, ctypes.c_uint32, ctypes.POINTER(vp), vp, vp]
        L.zero_ipc_export.restype = st
        L.zero_ipc_export.argtypes = [vp, ctypes.POINTER(_IpcHandle)]
        L.zero_ipc_open.restype = st
        L.zero_ipc_open.argtypes = [ctypes.POINTER(_IpcHandle), ctypes.POINTER(vp)]
        L.zero_ipc_close.restype = st
        L.zero_ipc_close.argtypes = [vp]
        L.zero_status_str.restype = ctypes.c_char_p
        L.zero_status_str.argtypes = [ctypes.c_int]
        L.zero_last_error.restype = ctypes.c_char_p
        L.zero_last_error.argtypes = []
        L.zero_abi_version.restype = ctypes.c_uint32
        L.zero_abi_version.argtypes = []
        _LIB = L
    return _LIB


def _check(status):
    if status != ZERO_OK:
        L = lib()
        msg = L.zero_last_error().decode() or L.zero_status_str(status).decode()
        raise ZeroError(status, msg)


class Plan:
    """Owns a zero_plan_t handle."""

    def __init__(self, handle):
        self._h = ctypes.c_void_p(handle)

    @property
    def handle(self):
        return self._h

    def query(self, what, idx=0):
        return zero_plan_query(self, what, idx)

    # convenience views of the plan
    @property
    def psi(self):
        return self.query(ZERO_Q_PSI)

    @property
    def psi_pad(self):
        return self.query(ZERO_Q_PSI_PAD)

    @property
    def S(self):
        return self.query(ZERO_Q_S)

    @property
    def nd(self):
        return self.query(ZERO_Q_ND)

    @property
    def stage(self):
        return self.query(ZERO_Q_STAGE)

    @property
    def n_units(self):
        return self.query(ZERO_Q_N_UNITS)

    @property
    def n_buckets(self):
        return self.query(ZERO_Q_N_BUCKETS)

    def units(self):
        """[(len, pad, shard, base, offset)] per unit."""
        return [tuple(self.query(q, u) for q in (ZERO_Q_UNIT_LEN, ZERO_Q_UNIT_PAD,
                                                  ZERO_Q_UNIT_SHARD, ZERO_Q_UNIT_BASE,
                                                  ZERO_Q_UNIT_OFFSET))
                for u in range(self.n_units)]

    def buckets(self):
        """[(unit, begin, end)] per bucket (logical, end exclusive)."""
        return [tuple(self.query(q, b) for q in (ZERO_Q_BUCKET_UNIT, ZERO_Q_BUCKET_BEGIN,
                                                  ZERO_Q_BUCKET_END))
                for b in range(self.n_buckets)]

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h and _LIB is not None:
            _LIB.zero_plan_destroy(h)


def zero_plan(psi, nd, stage, bucket_elems, align_elems=64, k_bytes=12,
              unit_elems=None, max_live=1):
    """Build a plan (see zero_plan in include/zero.h)."""
    desc = _PlanDesc()
    desc.psi = int(psi)
    desc.nd = int(nd)
    desc.stage = int(stage)
    desc.bucket_elems = int(bucket_elems)
    desc.align_elems = int(align_elems)
    desc.k_bytes = int(k_bytes)
    desc.max_live = int(max_live)
    arr = None
    if unit_elems:
        arr = (ctypes.c_uint64 * len(unit_elems))(*[int(x) for x in unit_elems])
        desc.n_units = len(unit_elems)
        desc.unit_elems = arr
    h = ctypes.c_void_p()
    _check(lib().zero_plan(ctypes.byref(desc), ctypes.byref(h)))
    return Plan(h.value)


def zero_plan_query(plan, what, idx=0):
    out = ctypes.c_uint64()
    _check(lib().zero_plan_query(plan.handle, int(what), int(idx), ctypes.byref(out)))
    return out.value


def zero_bytes_moved(plan, kind, flags=0):
    out = ctypes.c_uint64()
    _check(lib().zero_bytes_moved(plan.handle, int(kind), int(flags), ctypes.byref(out)))
    return out.value


def zero_release_layer(plan, unit):
    _check(lib().zero_release_layer(plan.handle, int(unit)))


# ------------------------------------------------------------ device calls
def _ptr(t, dtype=None, name="tensor"):
    """Device pointer of a CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    return t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _row_stride(t, default):
    if t is not None and t.dim() == 2:
        if t.stride(1) != 1:
            raise ValueError("rows must be contiguous")
        return t.stride(0)
    return default


def make_bufs(plan, grads, master, exp_avg, exp_avg_sq, params, reduced_grad=None,
              grad_norm_sq=None, overflow=None, workspace=None, owner_view=-1,
              grad_stride=None, param_stride=None, adam_consts=None):
    import torch
    b = _Bufs()
    b.grads = _ptr(grads, torch.bfloat16, "grads")
    default_g = plan.S if owner_view >= 0 else plan.psi_pad
    b.grad_stride = int(grad_stride if grad_stride is not None else _row_stride(grads, default_g))
    b.master = _ptr(master, torch.float32, "master")
    b.exp_avg = _ptr(exp_avg, torch.float32, "exp_avg")
    b.exp_avg_sq = _ptr(exp_avg_sq, torch.float32, "exp_avg_sq")
    b.params = _ptr(params, torch.bfloat16, "params")
    b.param_stride = int(param_stride if param_stride is not None
                         else _row_stride(params, plan.psi_pad))
    b.reduced_grad = _ptr(reduced_grad, torch.float32, "reduced_grad")
    b.grad_norm_sq = _ptr(grad_norm_sq, torch.float64, "grad_norm_sq")
    b.overflow = _ptr(overflow, torch.int32, "overflow")
    b.workspace = _ptr(workspace, None, "workspace")
    b.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    b.owner_view = int(owner_view)
    b.adam_consts = _ptr(adam_consts, torch.float32, "adam_consts")
    return b


def make_adam(adam):
    a = _Adam()
    a.lr = float(adam["lr"])
    a.beta1 = float(adam["beta1"])
    a.beta2 = float(adam["beta2"])
    a.eps = float(adam["eps"])
    a.grad_scale = float(adam["grad_scale"])
    a.weight_decay = float(adam.get("weight_decay", 0.0))
    return a


def zero_step(plan, grads, master, exp_avg, exp_avg_sq, params, adam, t, stream=None, **kw):
    """One full step (all buckets, then the optional norm/overflow)."""
    b = make_bufs(plan, grads, master, exp_avg, exp_avg_sq, params, **kw)
    _check(lib().zero_step(plan.handle, ctypes.byref(b), ctypes.byref(make_adam(adam)),
                           int(t), _stream(stream)))


def zero_step_noalloc(plan, grads, master, exp_avg, exp_avg_sq, params, adam, t, stream=None,
                      **kw):
    """zero_step without a workspace argument: the norm/overflow scratch is the
    library's own static device array (for callers that cannot allocate)."""
    if "workspace" in kw:
        raise ValueError("zero_step_noalloc takes no workspace")
    b = make_bufs(plan, grads, master, exp_avg, exp_avg_sq, params, **kw)
    _check(lib().zero_step_noalloc(plan.handle, ctypes.byref(b), ctypes.byref(make_adam(adam)),
                                   int(t), _stream(stream)))


def zero_step_guarded(plan, grads, master, exp_avg, exp_avg_sq, params, adam, t,
                      max_grad_norm=0.0, skip_nonfinite=True, stream=None, **kw):
    """The two-pass step with global-norm clipping and/or skipping on
    non-finite gradients (reduced_grad, grad_norm_sq, overflow and workspace
    are required keyword arguments)."""
    b = make_bufs(plan, grads, master, exp_avg, exp_avg_sq, params, **kw)
    g = _Guard()
    g.max_grad_norm = float(max_grad_norm)
    g.skip_nonfinite = 1 if skip_nonfinite else 0
    _check(lib().zero_step_guarded(plan.handle, ctypes.byref(b), ctypes.byref(make_adam(adam)),
                                   ctypes.byref(g), int(t), _stream(stream)))


def zero_step_buckets(plan, grads, master, exp_avg, exp_avg_sq, params, adam, t,
                      first_bucket, n_buckets, stream=None, **kw):
    """Buckets [first_bucket, first_bucket + n_buckets) of step t."""
    b = make_bufs(plan, grads, master, exp_avg, exp_avg_sq, params, **kw)
    _check(lib().zero_step_buckets(plan.handle, ctypes.byref(b), ctypes.byref(make_adam(adam)),
                                   int(t), int(first_bucket), int(n_buckets), _stream(stream)))


def zero_gather_layer(plan, unit, owner_params, full_layer, stream=None):
    import torch
    _check(lib().zero_gather_layer(plan.handle, int(unit),
                                   _ptr(owner_params, torch.bfloat16, "owner_params"),
                                   _ptr(full_layer, torch.bfloat16, "full_layer"),
                                   _stream(stream)))


ZERO_KERNEL_NONE = 0
ZERO_KERNEL_BULK_COPY = 1
ZERO_KERNEL_VECTOR_LOAD = 2


def zero_step_kernel(plan, owner_view=-1):
    """Name of the kernel zero_step uses for aligned bucket bodies on the
    current device: 'k_step_tma' (bulk-copy ring) or 'k_step_vec8'."""
    out = ctypes.c_uint32()
    _check(lib().zero_step_kernel(plan.handle, int(owner_view), ctypes.byref(out)))
    return "k_step_tma" if out.value == ZERO_KERNEL_BULK_COPY else "k_step_vec8"


def zero_step_peers_kernel(plan, rank, first=0, count=None):
    """Which kernel zero_step_peers runs rank's aligned bodies in, over
    buckets [first, first + count) (default: the whole step):
    "k_step_tma" (bulk copies through the peer table), "k_step_peer"
    (16-byte loads), or None when the call has no aligned body."""
    if count is None:
        count = plan.n_buckets - first
    out = ctypes.c_uint32()
    _check(lib().zero_step_peers_kernel(plan.handle, int(rank), int(first), int(count), ctypes.byref(out)))
    return {ZERO_KERNEL_BULK_COPY: "k_step_tma", ZERO_KERNEL_VECTOR_LOAD: "k_step_peer"}.get(out.value)


def zero_adam_consts(adam, t, out):
    """Fill `out` (a float32 tensor of >= 9 elements on the host) with step t's
    nine fp32 constants."""
    import torch
    if out.dtype != torch.float32 or out.numel() < 9 or out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous host float32 tensor of >= 9 elements")
    _check(lib().zero_adam_consts(ctypes.byref(make_adam(adam)), int(t),
                                  ctypes.c_void_p(out.data_ptr())))


def zero_stream_status(stream=None):
    """Synchronise the stream; raise ZeroError(ZERO_ETIMEOUT) if a bounded
    wait in the bulk-copy kernel gave up since the last check."""
    _check(lib().zero_stream_status(_stream(stream)))


def zero_reshard(from_plan, src, to_plan, dst, stream=None):
    """Copy one owner-storage state array (fp32 or bf16 tensor) from
    `from_plan`'s layout to `to_plan`'s (same units, other Nd or padding)."""
    import torch
    if src.dtype != dst.dtype or src.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("src and dst must both be float32 or both bfloat16")
    _check(lib().zero_reshard(from_plan.handle, _ptr(src, None, "src"), to_plan.handle,
                              _ptr(dst, None, "dst"), src.element_size(), _stream(stream)))


def workspace_for(plan, device="cuda"):
    """A caller-owned device workspace of the size the norm/overflow needs."""
    import torch
    return torch.empty(plan.query(ZERO_Q_WORKSPACE_BYTES), dtype=torch.uint8, device=device)


# ------------------------------------------------------ ranks as devices
def _dev_ptr(x, dtype, name):
    """A device pointer from a CUDA tensor or an int address (a peer mapping
    from zero_ipc_open); None -> NULL."""
    if x is None or isinstance(x, int):
        return x
    return _ptr(x, dtype, name)


def _ptr_array(items, dtype, name):
    arr = (ctypes.c_void_p * len(items))()
    for q, x in enumerate(items):
        arr[q] = _dev_ptr(x, dtype, "%s[%d]" % (name, q))
    return arr


def zero_step_peers(plan, rank, grads, params, master, exp_avg, exp_avg_sq, adam, t,
                    first_bucket=0, n_buckets=None, stream=None, reduced_grad=None,
                    grad_norm_sq=None, overflow=None, workspace=None, adam_consts=None):
    """Rank `rank`'s part of a step whose ranks have their own buffers.

    grads: Nd bf16 gradients [psi_pad] (CUDA tensors, or int addresses of peer
    mappings), one per rank.  params: Nd bf16 replicas [psi_pad] at stages
    1-2; at stage 3 only params[rank] (this rank's owner shard [S]) is used.
    master / exp_avg / exp_avg_sq: this rank's fp32 shard [S].
    """
    import torch
    nd = plan.nd
    if len(grads) != nd or len(params) != nd:
        raise ValueError("grads and params must hold one entry per rank (%d)" % nd)
    g_arr = _ptr_array(grads, torch.bfloat16, "grads")
    p_arr = _ptr_array(params, torch.bfloat16, "params")
    b = _PeerBufs()
    b.rank = int(rank)
    b.grads = ctypes.cast(g_arr, ctypes.POINTER(ctypes.c_void_p))
    b.params = ctypes.cast(p_arr, ctypes.POINTER(ctypes.c_void_p))
    b.master = _ptr(master, torch.float32, "master")
    b.exp_avg = _ptr(exp_avg, torch.float32, "exp_avg")
    b.exp_avg_sq = _ptr(exp_avg_sq, torch.float32, "exp_avg_sq")
    b.reduced_grad = _ptr(reduced_grad, torch.float32, "reduced_grad")
    b.grad_norm_sq = _ptr(grad_norm_sq, torch.float64, "grad_norm_sq")
    b.overflow = _ptr(overflow, torch.int32, "overflow")
    b.workspace = _ptr(workspace, None, "workspace")
    b.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    b.adam_consts = _ptr(adam_consts, torch.float32, "adam_consts")
    n = plan.n_buckets - int(first_bucket) if n_buckets is None else int(n_buckets)
    _check(lib().zero_step_peers(plan.handle, ctypes.byref(b), ctypes.byref(make_adam(adam)),
                                 int(t), int(first_bucket), n, _stream(stream)))


def zero_gather_layer_peers(plan, unit, owner_params, full_layer, stream=None):
    """Stage 3: materialise unit `unit` from the Nd owners' bf16 shards
    (tensors or int addresses of peer mappings), in rank order."""
    import torch
    if len(owner_params) != plan.nd:
        raise ValueError("owner_params must hold one entry per rank (%d)" % plan.nd)
    arr = _ptr_array(owner_params, torch.bfloat16, "owner_params")
    _check(lib().zero_gather_layer_peers(plan.handle, int(unit),
                                         ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)),
                                         _ptr(full_layer, torch.bfloat16, "full_layer"),
                                         _stream(stream)))


def zero_ipc_export(tensor_or_ptr):
    """IPC handle (bytes, IPC_HANDLE_BYTES long) of a CUDA buffer, to send to
    another process on the node."""
    h = _IpcHandle()
    p = tensor_or_ptr if isinstance(tensor_or_ptr, int) else _ptr(tensor_or_ptr, None, "buffer")
    _check(lib().zero_ipc_export(ctypes.c_void_p(p), ctypes.byref(h)))
    return bytes(h)


def zero_ipc_open(handle):
    """Map a buffer exported by another process (bytes from zero_ipc_export)
    on the current CUDA device; returns its address as an int."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle is %d bytes" % IPC_HANDLE_BYTES)
    h = _IpcHandle.from_buffer_copy(handle)
    out = ctypes.c_void_p()
    _check(lib().zero_ipc_open(ctypes.byref(h), ctypes.byref(out)))
    return int(out.value)


def zero_ipc_close(ptr):
    """Undo one zero_ipc_open()."""
    _check(lib().zero_ipc_close(ctypes.c_void_p(int(ptr))))
