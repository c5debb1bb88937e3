"""ctypes binding of libttt_b200.so (the C ABI declared in include/ttt.h).

Argument marshalling only: every step of the TTT forward pass runs in the CUDA
library.  torch tensors are used for device memory and streams.  There is no
CPU fallback: if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libttt_b200.so")

TTT_OK = 0
TTT_ERR_INVALID_ARG = -1
TTT_ERR_UNSUPPORTED = -2
TTT_ERR_CUDA = -3
TTT_ERR_NONFINITE = -4
TTT_ERR_TIMEOUT = -5
TTT_ERR_WORKSPACE = -6

INNER = {"linear": 0, "mlp2_gelu": 1, "swiglu": 2, "dwconv": 3, "glu": 4}
LOSS = {"mse": 0, "neg_dot": 1, "rmse": 2}
OPT = {"gd": 0, "momentum": 1, "muon": 2, "momentum_muon": 3}
DTYPE = {"f32": 0, "bf16": 1}
FLAG_KEY_INSTNORM = 1
FLAG_WEIGHT_L2NORM = 2
FLAG_DIRECT_LAUNCH = 4
FLAG_SINGLE_CTA = 8
FLAG_W0_PER_BATCH = 16
FLAG_NO_UPDATE = 32
FLAG_FIRST_LAYER_ONLY = 64

EXPORTED = [
    "ttt_config_init", "ttt_create", "ttt_param_count", "ttt_workspace_size", "ttt_forward",
    "ttt_host_staging_size", "ttt_forward_host", "ttt_query_status", "ttt_destroy", "ttt_status_string",
    "ttt_selftest_gemm", "ttt_profile_enable", "ttt_profile_collect", "ttt_stage_name", "ttt_launch_count",
    "ttt_forward_noalloc", "ttt_token_pair_capacity", "ttt_selftest_timeout", "ttt_plan_info",
    "ttt_state_size", "ttt_forward_state", "ttt_selftest_activation", "ttt_pair_schedule",
]
NUM_STAGES = 8


class TTTConfig(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("Nq", ctypes.c_int32),
        ("d", ctypes.c_int32), ("h", ctypes.c_int32), ("chunk", ctypes.c_int32), ("causal", ctypes.c_int32),
        ("inner", ctypes.c_int32), ("loss", ctypes.c_int32), ("opt", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("flags", ctypes.c_uint32), ("eta_scalar", ctypes.c_float), ("lr", ctypes.c_float),
        ("momentum", ctypes.c_float), ("ns_iters", ctypes.c_int32), ("ns_coeff", ctypes.c_float * 3),
        ("in_eps", ctypes.c_float), ("epochs", ctypes.c_int32),
        ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32), ("ksize", ctypes.c_int32),
    ]


class TTTError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} ({status})")
        self.status = status


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"CUDA library {_LIB_PATH} is missing: build it with weight_sequence_mixing_b200.build")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    cfgp = ctypes.POINTER(TTTConfig)
    sig = {
        "ttt_config_init": (None, [cfgp]),
        "ttt_create": (i32, [cfgp, ctypes.POINTER(vp)]),
        "ttt_param_count": (i64, [vp]),
        "ttt_workspace_size": (sz, [vp]),
        "ttt_forward": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ttt_host_staging_size": (sz, [vp]),
        "ttt_forward_host": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, sz, vp]),
        "ttt_query_status": (i32, [vp, vp, vp]),
        "ttt_destroy": (None, [vp]),
        "ttt_status_string": (ctypes.c_char_p, [i32]),
        "ttt_selftest_gemm": (i32, [i32] * 9 + [vp, vp, vp, vp]),
        "ttt_profile_enable": (i32, [vp, i32]),
        "ttt_profile_collect": (i32, [vp, i32, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)]),
        "ttt_stage_name": (ctypes.c_char_p, [i32]),
        "ttt_launch_count": (i64, [vp]),
        "ttt_forward_noalloc": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "ttt_token_pair_capacity": (i32, [i32]),
        "ttt_selftest_timeout": (i32, [vp, vp]),
        "ttt_selftest_activation": (i32, [i32, i64, vp, vp, vp, vp]),
        "ttt_pair_schedule": (i32, [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, i64]),
        "ttt_plan_info": (i32, [vp, ctypes.POINTER(ctypes.c_int), i32]),
        "ttt_state_size": (sz, [vp]),
        "ttt_forward_state": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def status_string(status: int) -> str:
    return LIB.ttt_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != TTT_OK:
        raise TTTError(status, where)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_config(cfg: dict) -> TTTConfig:
    """C config from a workload dict (see synth_inputs.make_config for the keys)."""
    c = TTTConfig()
    LIB.ttt_config_init(ctypes.byref(c))
    c.B, c.H, c.N, c.Nq = cfg["B"], cfg["H"], cfg["N"], cfg["Nq"]
    c.d, c.h = cfg["d"], cfg["h"]
    c.chunk, c.causal = int(cfg["chunk"] or 0), int(cfg["causal"])
    c.inner, c.loss, c.opt = INNER[cfg["inner"]], LOSS[cfg["loss"]], OPT[cfg["opt"]]
    c.dtype = DTYPE[cfg["dtype"]]
    c.flags = ((FLAG_KEY_INSTNORM if cfg["key_instnorm"] else 0) | (FLAG_WEIGHT_L2NORM if cfg["weight_l2norm"] else 0)
               | (FLAG_DIRECT_LAUNCH if cfg.get("direct_launch") else 0)
               | (FLAG_SINGLE_CTA if cfg.get("single_cta") else 0)
               | (FLAG_W0_PER_BATCH if cfg.get("w0_per_batch") else 0)
               | (FLAG_NO_UPDATE if cfg.get("no_update") else 0)
               | (FLAG_FIRST_LAYER_ONLY if cfg.get("first_layer_only") else 0))
    c.eta_scalar = float(cfg["eta_scalar"])
    c.lr = float(cfg["lr"])
    c.momentum = float(cfg["momentum"])
    c.ns_iters = int(cfg["ns_iters"])
    for i in range(3):
        c.ns_coeff[i] = float(cfg["ns_coeff"][i])
    c.in_eps = float(cfg["in_eps"])
    c.epochs = int(cfg.get("epochs", 1))
    c.grid_h = int(cfg.get("grid_h", 0))
    c.grid_w = int(cfg.get("grid_w", 0))
    c.ksize = int(cfg.get("ksize", 3))
    return c


@dataclass
class TTTLayer:
    """One configured TTT layer: a C handle plus its device workspace."""
    cfg: dict
    device: str = "cuda"
    _handle: ctypes.c_void_p = field(default=None, repr=False)
    workspace: torch.Tensor = field(default=None, repr=False)

    def __post_init__(self):
        self._c = make_config(self.cfg)
        h = ctypes.c_void_p()
        _check(LIB.ttt_create(ctypes.byref(self._c), ctypes.byref(h)), "ttt_create")
        self._handle = h
        self.P = int(LIB.ttt_param_count(h))
        ws = int(LIB.ttt_workspace_size(h))
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=self.device)

    def close(self):
        if self._handle:
            LIB.ttt_destroy(self._handle)
            self._handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def io_dtype(self):
        return torch.float32 if self.cfg["dtype"] == "f32" else torch.bfloat16

    def check_buffers(self, device_type: str, **bufs):
        """Element counts, dtypes and layout of a call's buffers: the library reads and
        writes them by the configured sizes, so a short buffer is refused here."""
        c = self.cfg
        BH = c["B"] * c["H"]
        q = BH * c["Nq"] * c["d"]
        kv = BH * c["N"] * c["d"]
        want = {"Q": (q, self.io_dtype), "K": (kv, self.io_dtype), "V": (kv, self.io_dtype),
                "eta": (BH * c["N"], torch.float32),
                "W0": ((BH if c.get("w0_per_batch") else c["H"]) * self.P, torch.float32),
                "O": (q, self.io_dtype), "W_out": (BH * self.P, torch.float32)}
        for name, t in bufs.items():
            if t is None:
                if name in ("Q", "K", "V", "W0", "O"):
                    raise ValueError(f"{name} is required")
                continue
            n, dt = want[name]
            if t.numel() != n or t.dtype != dt:
                raise ValueError(f"{name}: expected {n} elements of {dt}, got shape {tuple(t.shape)} of {t.dtype}")
            if not t.is_contiguous() or t.device.type != device_type:
                raise ValueError(f"{name}: must be a contiguous {device_type} tensor")

    def forward(self, Q, K, V, eta, W0, O=None, W_out=None, stream=None, check=True):
        """Enqueue the layer on `stream`; returns (O, W_out).  With check=True the
        stream is synchronised and the device status word is checked."""
        c = self.cfg
        if O is None:
            O = torch.empty((c["B"], c["H"], c["Nq"], c["d"]), dtype=self.io_dtype, device=self.device)
        if W_out is None:
            W_out = torch.empty((c["B"], c["H"], self.P), dtype=torch.float32, device=self.device)
        self.check_buffers("cuda", Q=Q, K=K, V=V, eta=eta, W0=W0, O=O, W_out=W_out)
        st = _stream_ptr(stream)
        _check(LIB.ttt_forward(self._handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0), _ptr(O), _ptr(W_out),
                               _ptr(self.workspace), self.workspace.numel(), st), "ttt_forward")
        if check:
            self.check_status(stream)
        return O, W_out

    @property
    def state_size(self) -> int:
        """Bytes of the momentum state a call hands on (0 without momentum)."""
        return int(LIB.ttt_state_size(self._handle))

    def new_state(self):
        """A device buffer for the momentum state (at least 16 bytes)."""
        return torch.zeros(max(self.state_size, 16), dtype=torch.uint8, device=self.device)

    def forward_state(self, Q, K, V, eta, W0, state_in=None, state_out=None, O=None, W_out=None, stream=None,
                      check=True):
        """As forward, carrying the momentum state in (state_in, or None: zero) and out
        (state_out, or None); both uint8 device buffers of at least state_size bytes."""
        c = self.cfg
        if O is None:
            O = torch.empty((c["B"], c["H"], c["Nq"], c["d"]), dtype=self.io_dtype, device=self.device)
        if W_out is None:
            W_out = torch.empty((c["B"], c["H"], self.P), dtype=torch.float32, device=self.device)
        self.check_buffers("cuda", Q=Q, K=K, V=V, eta=eta, W0=W0, O=O, W_out=W_out)
        for t in (state_in, state_out):
            if t is not None and (t.numel() * t.element_size() < self.state_size or t.device.type != "cuda"):
                raise ValueError("state buffer smaller than state_size or not on the GPU")
        st = _stream_ptr(stream)
        _check(LIB.ttt_forward_state(self._handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0), _ptr(O),
                                     _ptr(W_out), _ptr(state_in), _ptr(state_out), _ptr(self.workspace),
                                     self.workspace.numel(), st), "ttt_forward_state")
        if check:
            self.check_status(stream)
        return O, W_out

    def check_status(self, stream=None):
        _check(LIB.ttt_query_status(self._handle, _ptr(self.workspace), _stream_ptr(stream)), "device status")

    def forward_noalloc(self, Q, K, V, eta, W0, O, W_out=None, status=None, stream=None):
        """The layer without a workspace argument: the library's own static device
        scratch stands in for it (for callers that cannot allocate; see ttt.h)."""
        self.check_buffers("cuda", Q=Q, K=K, V=V, eta=eta, W0=W0, O=O, W_out=W_out)
        _check(LIB.ttt_forward_noalloc(self._handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0), _ptr(O),
                                       _ptr(W_out), _ptr(status), _stream_ptr(stream)), "ttt_forward_noalloc")

    # ---- per-stage device timing (CUDA events around every launch, on its stream)
    def profile(self, on: bool):
        _check(LIB.ttt_profile_enable(self._handle, int(bool(on))), "ttt_profile_enable")

    def profile_collect(self) -> dict:
        ms = (ctypes.c_float * NUM_STAGES)()
        cnt = (ctypes.c_int * NUM_STAGES)()
        _check(LIB.ttt_profile_collect(self._handle, NUM_STAGES, ms, cnt), "ttt_profile_collect")
        return {LIB.ttt_stage_name(i).decode(): (float(ms[i]), int(cnt[i])) for i in range(NUM_STAGES) if cnt[i]}

    def launch_count(self) -> int:
        return int(LIB.ttt_launch_count(self._handle))

    # ---- host-buffer entry point (copies inside the library call)
    def staging(self):
        n = int(LIB.ttt_host_staging_size(self._handle))
        return torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)

    def forward_host(self, Q, K, V, eta, W0, O, W_out, staging, stream=None):
        """Host (ideally pinned) CPU tensors in and out; enqueued on `stream`."""
        self.check_buffers("cpu", Q=Q, K=K, V=V, eta=eta, W0=W0, O=O, W_out=W_out)
        if staging.numel() < int(LIB.ttt_host_staging_size(self._handle)) or staging.device.type != "cuda":
            raise ValueError("staging must be a device buffer of at least ttt_host_staging_size bytes")
        st = _stream_ptr(stream)
        _check(LIB.ttt_forward_host(self._handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0), _ptr(O),
                                    _ptr(W_out), _ptr(staging), staging.numel(), _ptr(self.workspace),
                                    self.workspace.numel(), st), "ttt_forward_host")


def selftest_gemm(A, B, elem_bytes, a_mn, b_mn, bn, M, N, K, batches, splits, stream=None):
    """Diagnostic: C[s][z] = A[z] B[z]^T through the tcgen05 engine (see ttt_diag.h)."""
    C = torch.full((splits, batches, M, N), float("nan"), dtype=torch.float32, device=A.device)
    _check(LIB.ttt_selftest_gemm(elem_bytes, int(a_mn), int(b_mn), bn, M, N, K, batches, splits, _ptr(A), _ptr(B),
                                 _ptr(C), _stream_ptr(stream)), "ttt_selftest_gemm")
    return C


def token_pair_capacity(swiglu: bool) -> int:
    """CTA pairs of the token-phase kernel resident at once on the current device (0: single-CTA fallback)."""
    return int(LIB.ttt_token_pair_capacity(int(bool(swiglu))))


def pair_schedule(m_tiles: int, n_tiles: int, batches: int, kblocks: int, cap_resident: int,
                  cap_streaming: int) -> tuple[bool, int, list[int], list[tuple[int, int, int]]]:
    """The token phase's CTA-pair tile schedule (host logic; see ttt_diag.h): (resident form,
    pairs, tiles per pair, (head, token tile, hidden block) of every tile pair by pair)."""
    total = m_tiles * n_tiles * batches
    counts = (ctypes.c_int * max(cap_resident, cap_streaming, 1))()
    tiles = (ctypes.c_int * (3 * max(total, 1)))()
    res, pairs = ctypes.c_int(), ctypes.c_int()
    n = LIB.ttt_pair_schedule(m_tiles, n_tiles, batches, kblocks, cap_resident, cap_streaming, ctypes.byref(res),
                              ctypes.byref(pairs), counts, tiles, total)
    if n < 0:
        raise TTTError(n, "ttt_pair_schedule")
    return bool(res.value), pairs.value, list(counts[:pairs.value]), [tuple(tiles[3 * i:3 * i + 3]) for i in range(n)]


def selftest_timeout(status_word: torch.Tensor, stream=None) -> int:
    """Status (TTT_ERR_TIMEOUT expected) of a kernel whose bounded wait runs out; see ttt_diag.h."""
    return int(LIB.ttt_selftest_timeout(_ptr(status_word), _stream_ptr(stream)))


def selftest_activation(kind: str, x: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """The epilogues' activation ("gelu" or "silu") and its derivative, or the apply's GELU alone
    ("gelu_fwd", derivative 0), on fp32 device values; see ttt_diag.h."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    y, dy = torch.empty_like(x), torch.empty_like(x)
    _check(LIB.ttt_selftest_activation({"gelu": 0, "silu": 1, "gelu_fwd": 2}[kind], x.numel(), _ptr(x), _ptr(y), _ptr(dy),
                                       _stream_ptr(stream)), "ttt_selftest_activation")
    return y, dy


PLAN_FIELDS = ("path", "chunk", "nchunks", "splits", "tile_rows", "grad_bn", "direct")


def plan_info(cfg: dict) -> dict:
    """The execution plan ttt_create chooses for `cfg` (host logic; no GPU needed)."""
    c = make_config(cfg)
    h = ctypes.c_void_p()
    _check(LIB.ttt_create(ctypes.byref(c), ctypes.byref(h)), "ttt_create")
    try:
        buf = (ctypes.c_int * len(PLAN_FIELDS))()
        n = LIB.ttt_plan_info(h, buf, len(PLAN_FIELDS))
        if n < 0:
            raise TTTError(n, "ttt_plan_info")
        return dict(zip(PLAN_FIELDS, list(buf)[:n]))
    finally:
        LIB.ttt_destroy(h)
