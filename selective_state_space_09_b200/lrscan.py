"""Thin Python binding of the C ABI in ``include/lrscan.h`` (argument marshalling only).

Every step of the scan runs in the CUDA library ``_lrscan.so``; this module only builds the
descriptor and pointer structs from torch tensors and passes torch's current CUDA stream.  torch
supplies device memory and streams, nothing else.  Importing it without the built library raises
``ImportError``: there is no CPU fallback.

Layouts and dtypes are those of the header (token-major, row-major).  ``Plan`` holds the
checkpoint buffer and workspace of one problem so that repeated calls allocate nothing.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lrscan.so")
if not os.path.exists(LIB_PATH):
    raise ImportError("CUDA scan library %s is not built (run selective_state_space_09_b200/build.py "
                      "or __graft_entry__.build())" % LIB_PATH)

KIND = {"rglru": 0, "rotlru": 1, "s6": 2, "ssd": 3, "gla": 4}
DISC = {"none": 0, "zoh": 1, "bilinear": 2, "dirac": 3, "zoh_euler": 4}
IO = {torch.float32: 0, torch.bfloat16: 1}
HAS_Z, HAS_DSKIP, FULL_STATE, DELTA_SOFTPLUS, RGLRU_GATES = 1, 2, 4, 8, 16
# test hooks (lrscan.h): withheld carry (timeout path), widest SSD head blocks
TEST_WITHHOLD_CARRY, TEST_MAX_HEAD_BLOCK, TEST_LOOKBACK = 0x80000000, 0x40000000, 0x20000000
STATUS = ["ok", "invalid argument", "unsupported by this library", "misaligned pointer or innermost extent",
          "workspace too small", "CUDA runtime error", "device wait timed out",
          "device consistency check failed"]


class LrScanError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = int(status)
        msg = lib.lr_status_string(self.status).decode()
        super().__init__("%s: %s (status %d)" % (where, msg, self.status))


class Desc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("disc", ctypes.c_int32), ("io", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("B", ctypes.c_int64), ("L", ctypes.c_int64),
                ("D", ctypes.c_int64), ("H", ctypes.c_int64), ("P", ctypes.c_int64),
                ("N", ctypes.c_int64), ("G", ctypes.c_int64), ("chunk", ctypes.c_int32),
                ("segment", ctypes.c_int32)]


_IN = ["a", "b", "g", "mag", "theta", "x", "delta", "A", "Bm", "Cm", "Dskip", "z", "q", "k", "v",
       "delta_bias"]
_GR = ["da", "db", "dg", "dmag", "dtheta", "dx", "ddelta", "dA", "dBm", "dCm", "dDskip", "dz",
       "dq", "dk", "dv", "ddelta_bias"]


class Inputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _IN]


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _GR]


def _load():
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    pd = ctypes.POINTER(Desc)
    L.lr_validate.argtypes = [pd]
    L.lr_validate.restype = st
    L.lr_ckpt_bytes.argtypes = [pd]
    L.lr_ckpt_bytes.restype = sz
    L.lr_workspace_bytes.argtypes = [pd, ctypes.c_int]
    L.lr_workspace_bytes.restype = sz
    L.lr_scan_fwd.argtypes = [pd, ctypes.POINTER(Inputs), vp, vp, vp, sz, vp]
    L.lr_scan_fwd.restype = st
    L.lr_scan_bwd.argtypes = [pd, ctypes.POINTER(Inputs), vp, vp, ctypes.POINTER(Grads), vp, sz, vp]
    L.lr_scan_bwd.restype = st
    L.lr_get_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
    L.lr_get_error.restype = st
    L.lr_status_string.argtypes = [st]
    L.lr_status_string.restype = ctypes.c_char_p
    L.lr_last_dispatch.restype = ctypes.c_char_p
    L.lr_last_launch_count.restype = ctypes.c_int
    L.lr_set_launch_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
    L.lr_set_launch_events.restype = None
    L.lr_version.restype = ctypes.c_int
    L.lr_step.argtypes = [pd, ctypes.POINTER(Inputs), vp, vp, vp, vp]
    L.lr_step.restype = st
    L.lr_probe_pipe.argtypes = [ctypes.c_int, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
    L.lr_probe_pipe.restype = ctypes.c_int64
    return L


lib = _load()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def make_desc(kind, io=torch.float32, B=1, L=1, D=0, H=0, P=0, N=0, G=0, segment=1, chunk=0,
              disc="none", has_z=False, has_d=False):
    return Desc(KIND[kind], DISC[disc], IO[io], (HAS_Z if has_z else 0) | (HAS_DSKIP if has_d else 0),
                B, L, D, H, P, N, G, chunk, segment)


def validate(desc):
    return int(lib.lr_validate(ctypes.byref(desc)))


def ckpt_bytes(desc):
    return int(lib.lr_ckpt_bytes(ctypes.byref(desc)))


def workspace_bytes(desc, backward):
    return int(lib.lr_workspace_bytes(ctypes.byref(desc), 1 if backward else 0))


def last_dispatch():
    return lib.lr_last_dispatch().decode()


def last_launch_count():
    return int(lib.lr_last_launch_count())


def set_launch_events(events):
    """Timing hook: each kernel launch of the following calls on this thread first records
    events[k] (torch.cuda.Event, already created) on the call's stream; None turns it off."""
    if not events:
        lib.lr_set_launch_events(None, 0)
        set_launch_events._keep = None
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    set_launch_events._keep = arr  # the library keeps the pointer until the hook is reset
    lib.lr_set_launch_events(arr, len(events))


def probe_pipe(which, out, blocks, threads, iters):
    """lr_probe_pipe: one launch that keeps the special-function unit (which = "ex2") or the fp32
    FMA pipe (which = "ffma") busy; out: f32 device tensor of blocks * threads elements.  Returns
    the number of results the launch produces."""
    assert out.numel() >= blocks * threads and out.dtype == torch.float32 and out.is_cuda
    n = int(lib.lr_probe_pipe({"ex2": 0, "ffma": 1}[which], _ptr(out), blocks, threads, iters, _stream()))
    if n < 0:
        raise LrScanError(1, "lr_probe_pipe")
    return n


def _check(status, where):
    if status != 0:
        raise LrScanError(status, where)


class Plan:
    """Checkpoint buffer and workspace of one problem, allocated once on ``device``."""

    def __init__(self, desc, device="cuda"):
        s = validate(desc)
        if s != 0:
            raise LrScanError(s, "lr_validate")
        self.desc = desc
        self.device = torch.device(device)
        nck = ckpt_bytes(desc)
        nws = max(workspace_bytes(desc, False), workspace_bytes(desc, True))
        self.ckpt = torch.empty(max(nck // 4, 4), dtype=torch.float32, device=self.device)
        self.ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=self.device)
        self.ws_bytes = self.ws.numel()

    def fwd(self, inp, y):
        """inp: dict of tensors named as in ``Inputs`` (a, b, g, mag, theta, x, delta, A, Bm,
        Cm, Dskip, z, q, k, v); y: output tensor (written)."""
        ii = Inputs(*[_ptr(inp.get(n)) for n in _IN])
        _check(lib.lr_scan_fwd(ctypes.byref(self.desc), ctypes.byref(ii), _ptr(y), _ptr(self.ckpt),
                               _ptr(self.ws), self.ws_bytes, _stream()), "lr_scan_fwd")
        return y

    def bwd(self, inp, dy, grads):
        """grads: dict of output tensors named as in ``Grads`` (written)."""
        ii = Inputs(*[_ptr(inp.get(n)) for n in _IN])
        gg = Grads(*[_ptr(grads.get(n)) for n in _GR])
        _check(lib.lr_scan_bwd(ctypes.byref(self.desc), ctypes.byref(ii), _ptr(dy), _ptr(self.ckpt),
                               ctypes.byref(gg), _ptr(self.ws), self.ws_bytes, _stream()), "lr_scan_bwd")
        return grads

    def device_error(self):
        """Synchronises and returns (status, info) of the device-side error record."""
        info = ctypes.c_int32(0)
        s = lib.lr_get_error(_ptr(self.ws), _stream(), ctypes.byref(info))
        return int(s), int(info.value)

    def ckpt_view(self):
        """The checkpoint buffer as an f32 tensor of ceil(L/S) states (L with FULL_STATE)."""
        d = self.desc
        nseg = d.L if d.flags & FULL_STATE else (d.L + d.segment - 1) // d.segment
        shapes = {0: (nseg, d.B, d.D), 1: (nseg, d.B, d.D), 2: (nseg, d.B, d.D, d.N),
                  3: (nseg, d.B, d.H, d.N, d.P), 4: (nseg, d.B, d.H, d.N, d.P)}
        shp = shapes[d.kind]
        n = 1
        for s in shp:
            n *= s
        return self.ckpt[:n].view(*shp)


# ------------------------------------------------------------------ per-kind convenience plans
def desc_for(kind, inp, segment=1, disc="none", chunk=0, delta_softplus=False, gates=False):
    """Descriptor of a kind from its input tensors (shapes read from the tensors).
    delta_softplus (S6, SSD): dt = softplus(delta + inp["delta_bias"]) in the kernels.
    gates (rglru): the RG-LRU gate front-end; inp["a"], inp["b"], inp["x"], inp["A"] hold the
    recurrence gate r, the input gate i, x and Lambda."""
    if kind == "rglru":
        B, L, D = inp["a"].shape
        d = make_desc("rglru", inp["a"].dtype, B, L, D=D, segment=segment)
    elif kind == "rotlru":
        B, L, D = inp["b"].shape
        d = make_desc("rotlru", inp["b"].dtype, B, L, D=D, segment=segment)
    elif kind == "s6":
        B, L, D = inp["x"].shape
        N = inp["A"].shape[1]
        d = make_desc("s6", inp["x"].dtype, B, L, D=D, N=N, segment=segment, disc=disc,
                      has_z=inp.get("z") is not None, has_d=inp.get("Dskip") is not None)
    elif kind == "ssd":
        B, L, H, P = inp["x"].shape
        G, N = inp["Bm"].shape[2], inp["Bm"].shape[3]
        d = make_desc("ssd", inp["x"].dtype, B, L, H=H, P=P, N=N, G=G, segment=segment,
                      chunk=chunk, disc=disc, has_z=inp.get("z") is not None,
                      has_d=inp.get("Dskip") is not None)
    elif kind == "gla":
        B, L, H, K = inp["q"].shape
        V = inp["v"].shape[3]
        d = make_desc("gla", inp["q"].dtype, B, L, H=H, P=V, N=K, segment=segment, chunk=chunk)
    else:
        raise KeyError(kind)
    if delta_softplus:
        d.flags |= DELTA_SOFTPLUS
    if gates:
        d.flags |= RGLRU_GATES
    return d


def plan_for(kind, inp, segment, disc="none", chunk=0, delta_softplus=False, gates=False):
    """Build the Plan of a kind from its input tensors (shapes read from the tensors)."""
    d = desc_for(kind, inp, segment, disc, chunk, delta_softplus, gates)
    return Plan(d, inp[next(k for k in inp if inp[k] is not None)].device)


# ------------------------------------------------------------------------ decode / continuation
# per-token inputs of each kind (the rest are parameters)
TOKEN_INPUTS = {"rglru": ("a", "b", "x"), "rotlru": ("b", "g"), "s6": ("x", "delta", "Bm", "Cm", "z"),
                "ssd": ("x", "delta", "Bm", "Cm", "z"), "gla": ("q", "k", "v", "g")}


def state_shape(desc):
    """Shape of the f32 state lr_step reads and writes (see lrscan.h)."""
    d = desc
    return {0: (d.B, d.D), 1: (d.B, d.D), 2: (d.B, d.D, d.N), 3: (d.B, d.H, d.N, d.P),
            4: (d.B, d.H, d.N, d.P)}[d.kind]


def step(desc, inp, y, state_out, state_in=None):
    """lr_step: advance by desc.L steps from state_in (None: zero state) into state_out (may be
    state_in), writing the steps' outputs into y."""
    ii = Inputs(*[_ptr(inp.get(n)) for n in _IN])
    _check(lib.lr_step(ctypes.byref(desc), ctypes.byref(ii), _ptr(state_in), _ptr(state_out), _ptr(y),
                       _stream()), "lr_step")
    return y


class DecodeGraph:
    """T one-token steps captured once in a CUDA graph; ``replay()`` runs them all.

    ``seq``: the kind's inputs, token tensors time-major and contiguous, [T, B, 1, ...] (token t's
    inputs are ``seq[name][t]``), parameters as usual; ``state``: the f32 state, advanced in place;
    ``y``: [T, B, 1, ...] outputs.  Every replay continues from whatever ``state`` holds."""

    def __init__(self, kind, seq, state, y, disc="none", delta_softplus=False, gates=False):
        toks = TOKEN_INPUTS[kind]
        T = y.shape[0]
        self.kind, self.T, self.state, self.y = kind, T, state, y
        first = {n: (seq[n][0] if n in toks and seq.get(n) is not None else seq.get(n)) for n in seq}
        self.desc = desc_for(kind, first, 1, disc, delta_softplus=delta_softplus, gates=gates)
        self.calls = [({n: (seq[n][t] if n in toks and seq.get(n) is not None else seq.get(n)) for n in seq}, y[t])
                      for t in range(T)]
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # one eager step (on scratch buffers) settles lazy initialisation
            step(self.desc, self.calls[0][0], torch.empty_like(y[0]), state.clone(), state)
        torch.cuda.current_stream().wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            for inp, yt in self.calls:
                step(self.desc, inp, yt, state, state)

    def replay(self):
        self.graph.replay()


class StepGraph:
    """The forward and backward call of one training step of ``plan`` captured once in a CUDA
    graph; ``replay()`` runs both again on the same buffers (each kernel launch is then a node of
    one graph launch instead of a separate stream launch).  ``inp``, ``dy``, ``y`` and ``grads``
    are the tensors given here: write a step's inputs into them before a replay, read its results
    after.  The kernels and their work are those of ``plan.fwd`` / ``plan.bwd``."""

    def __init__(self, plan, inp, dy, y, grads):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # one eager step settles lazy initialisation
            plan.fwd(inp, y)
            plan.bwd(inp, dy, grads)
        torch.cuda.current_stream().wait_stream(side)
        self.plan = plan
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            plan.fwd(inp, y)
            plan.bwd(inp, dy, grads)

    def replay(self):
        self.graph.replay()


def alloc_outputs(kind, inp):
    """Output tensor and empty gradient tensors for a kind (shapes/dtypes of the header)."""
    e = torch.empty_like
    f32 = lambda t: torch.empty(t.shape, dtype=torch.float32, device=t.device)
    if kind == "rglru":
        g = {"da": e(inp["a"]), "db": e(inp["b"])}
        if inp.get("x") is not None:  # gate front-end: dx, dLambda
            g["dx"] = e(inp["x"])
            g["dA"] = e(inp["A"])
        return e(inp["b"]), g
    if kind == "rotlru":
        return e(inp["b"]), {"db": e(inp["b"]), "dg": e(inp["g"]), "dmag": e(inp["mag"]),
                             "dtheta": e(inp["theta"])}
    if kind in ("s6", "ssd"):
        g = {"dx": e(inp["x"]), "ddelta": e(inp["delta"]), "dA": e(inp["A"]), "dBm": f32(inp["Bm"]),
             "dCm": f32(inp["Cm"])}
        if inp.get("Dskip") is not None:
            g["dDskip"] = e(inp["Dskip"])
        if inp.get("z") is not None:
            g["dz"] = e(inp["z"])
        if inp.get("delta_bias") is not None:
            g["ddelta_bias"] = e(inp["delta_bias"])
        return e(inp["x"]), g
    if kind == "gla":
        return e(inp["v"]), {"dq": e(inp["q"]), "dk": e(inp["k"]), "dv": e(inp["v"]), "dg": e(inp["g"])}
    raise KeyError(kind)


# ---------------------------------------------------------------------- autograd wrappers
class _ScanFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, kind, names, segment, disc, chunk, opts, *tensors):
        inp = {n: t.contiguous() if t is not None else None for n, t in zip(names, tensors)}
        plan = plan_for(kind, inp, segment, disc, chunk, **opts)
        y, _ = alloc_outputs(kind, inp)
        plan.fwd(inp, y)
        ctx.kind, ctx.names, ctx.plan = kind, names, plan
        ctx.save_for_backward(*[inp[n] for n in names])
        return y

    @staticmethod
    def backward(ctx, dy):
        inp = dict(zip(ctx.names, ctx.saved_tensors))
        _, grads = alloc_outputs(ctx.kind, inp)
        ctx.plan.bwd(inp, dy.contiguous(), grads)
        out = []
        for n in ctx.names:
            t = inp[n]
            out.append(grads.get("d" + n) if t is not None else None)
        return (None, None, None, None, None, None) + tuple(out)


def rglru(a, b, segment=128):
    """y = rglru_scan(a, b): h_t = a_t h_{t-1} + b_t, y_t = h_t.  a, b: [B, L, D]."""
    return _ScanFn.apply("rglru", ("a", "b"), segment, "none", 0, {}, a, b)


def rglru_gated(r, i, x, lam, segment=128):
    """RG-LRU with its gates formed in the kernels: a = sigmoid(lam)^(8 r), b = sqrt(1 - a^2) (i x),
    h_t = a_t h_{t-1} + b_t, y_t = h_t.  r, i, x: [B, L, D] f32; lam: [D] f32.  Gradients flow to
    r, i, x and lam."""
    return _ScanFn.apply("rglru", ("a", "b", "x", "A"), segment, "none", 0, {"gates": True}, r, i, x, lam)


def rotlru(b, g, mag, theta, segment=256):
    """y = rotlru_scan: lambda_t = mag g_t e^{i theta}, h_t = lambda_t h_{t-1} + b_t (pairs)."""
    return _ScanFn.apply("rotlru", ("b", "g", "mag", "theta"), segment, "none", 0, {}, b, g, mag, theta)


def s6(x, delta, A, B, C, D=None, z=None, disc="zoh", segment=256, delta_softplus=False, delta_bias=None):
    """Selective scan S6 with fused D skip and silu(z) gate.  x, delta, z: [B, L, D].  With
    delta_softplus the step length is softplus(delta + delta_bias) (delta_bias [D] or None)."""
    return _ScanFn.apply("s6", ("x", "delta", "A", "Bm", "Cm", "Dskip", "z", "delta_bias"), segment, disc, 0,
                         {"delta_softplus": delta_softplus}, x, delta, A, B, C, D, z, delta_bias)


def ssd(x, delta, A, B, C, D=None, z=None, disc="zoh", chunk=64, segment=256, delta_softplus=False,
        delta_bias=None):
    """Head-wise SSD scan.  x, z: [B, L, H, P]; delta: [B, L, H]; B, C: [B, L, G, N].  With
    delta_softplus the step length is softplus(delta + delta_bias) (delta_bias [H] or None)."""
    return _ScanFn.apply("ssd", ("x", "delta", "A", "Bm", "Cm", "Dskip", "z", "delta_bias"), segment, disc,
                         chunk, {"delta_softplus": delta_softplus}, x, delta, A, B, C, D, z, delta_bias)


def gla(q, k, v, g, chunk=64, segment=256):
    """GLA scan: S_t = g_t S_{t-1} + k_t v_t^T, o_t = S_t^T q_t."""
    return _ScanFn.apply("gla", ("q", "k", "v", "g"), segment, "none", chunk, {}, q, k, v, g)
