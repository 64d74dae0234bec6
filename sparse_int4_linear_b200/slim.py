"""Python binding of libslim (ctypes; argument marshalling only).

Every step of the layer runs in the CUDA library; this module only allocates
device memory with torch, passes pointers, sizes and the current CUDA
stream, and turns status codes into exceptions.  There is no CPU or
PyTorch fallback: if libslim.so is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# SLIM_LIBRARY=debug loads the build with kernel index checks (libslim_debug.so).
DEBUG = os.environ.get("SLIM_LIBRARY", "") == "debug"
LIB_PATH = os.path.join(_PKG, "libslim_debug.so" if DEBUG else "libslim.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run `python -m sparse_int4_linear_b200.build` (needs nvcc)")

_lib = ctypes.CDLL(LIB_PATH)

c_int, c_size_t, c_void_p, c_char_p = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_char_p

STATUS = {
    0: "SLIM_OK", -1: "SLIM_ERR_ARG", -2: "SLIM_ERR_ALIGN", -3: "SLIM_ERR_SHAPE",
    -4: "SLIM_ERR_WORKSPACE", -5: "SLIM_ERR_RANGE", -6: "SLIM_ERR_TIMEOUT", -7: "SLIM_ERR_CUDA",
    -8: "SLIM_ERR_UNSUPPORTED", -9: "SLIM_ERR_STATE", -10: "SLIM_ERR_BOUNDS",
}
GROUP = 128
MAX_GROUPS = 8


class SlimLayerDesc(ctypes.Structure):
    _fields_ = [
        ("magic", ctypes.c_uint32),
        ("K", ctypes.c_int32), ("N", ctypes.c_int32), ("r", ctypes.c_int32), ("group", ctypes.c_int32),
        ("r16", ctypes.c_int32), ("n_groups", ctypes.c_int32), ("group_end", ctypes.c_int32 * 8),
        ("rl16", ctypes.c_int32), ("n_row_tiles", ctypes.c_int32), ("n_kblocks", ctypes.c_int32),
        ("base", c_void_p), ("bytes", c_size_t),
        ("vals", c_void_p), ("meta", c_void_p), ("scales", c_void_p), ("dec", c_void_p),
        ("Lf", c_void_p), ("Rf", c_void_p), ("Rp", c_void_p), ("Lp", c_void_p), ("status", c_void_p),
        ("Lq", c_void_p), ("Rq", c_void_p), ("adapter_bits", ctypes.c_int32),
    ]


_P = ctypes.POINTER(SlimLayerDesc)
_SIGS = {
    "slim_layer_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "slim_layer_init": (c_int, [_P, c_int, c_int, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "slim_grouped_layer_bytes": (c_size_t, [c_int, c_int, ctypes.POINTER(ctypes.c_int32), c_int, c_int]),
    "slim_grouped_layer_init": (c_int, [_P, c_int, c_int, ctypes.POINTER(ctypes.c_int32), c_int, c_int, c_void_p,
                                        c_size_t, c_void_p]),
    "slim_pack": (c_int, [_P, c_void_p, c_void_p, c_void_p, c_void_p]),
    "slim_layer_set_adapter_bits": (c_int, [_P, c_int]),
    "slim_unpack_adapters": (c_int, [_P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "slim_workspace_bytes": (c_size_t, [_P, c_int]),
    "slim_linear": (c_int, [_P, c_void_p, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "slim_host_workspace_bytes": (c_size_t, [_P, c_int]),
    "slim_linear_host": (c_int, [_P, c_void_p, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "slim_linear_host_async": (c_int, [_P, c_void_p, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "slim_unpack_dec": (c_int, [_P, c_void_p, c_void_p, c_void_p]),
    "slim_test_wait_timeout": (c_int, [_P, c_int, c_void_p]),
    "slim_test_stream_timeout": (c_int, [_P, c_void_p, c_int, c_void_p, c_void_p, c_size_t, c_int, c_void_p]),
    "slim_tuning_reload": (None, []),
    "slim_linear_noalloc": (c_int, [_P, c_void_p, c_int, c_void_p, c_void_p]),
    "slim_sync_status": (c_int, [_P, c_void_p]),
    "slim_status_string": (c_char_p, [c_int]),
    "slim_linear_launches": (c_int, [_P, c_int]),
    "slim_last_cuda_error": (c_int, []),
    "slim_abi_version": (c_int, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class SlimError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.name = STATUS.get(code, str(code))
        msg = _lib.slim_status_string(code).decode()
        if code == -7:
            msg += f" (cudaError {_lib.slim_last_cuda_error()})"
        super().__init__(f"{where}: {self.name}: {msg}")


def _check(code: int, where: str) -> None:
    if code != 0:
        raise SlimError(code, where)


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _as_bits(t: torch.Tensor, shape, name: str) -> torch.Tensor:
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"{name} must be bf16 (or its 16-bit pattern), got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return t.contiguous()


def layer_bytes(K: int, N: int, r: int) -> int:
    return int(_lib.slim_layer_bytes(K, N, r, GROUP))


def _n_array(N_list):
    return (ctypes.c_int32 * len(N_list))(*N_list)


class PackedLayer:
    """A packed layer: one device buffer plus its descriptor.  `N` is an int,
    or a list of row counts for a grouped layer that fuses several linears
    reading the same X (see slim_grouped_layer_init)."""

    def __init__(self, K: int, N, r: int, device=None, stream=None):
        N_list = [N] if isinstance(N, int) else list(N)
        nbytes = int(_lib.slim_grouped_layer_bytes(K, len(N_list), _n_array(N_list), r, GROUP))
        if nbytes == 0:
            raise SlimError(-3, "slim_grouped_layer_bytes")
        device = device or torch.device("cuda", torch.cuda.current_device())
        self.buf = torch.empty(nbytes + 1024, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 1024
        self._base = self.buf[off:off + nbytes]
        self.desc = SlimLayerDesc()
        _check(_lib.slim_grouped_layer_init(ctypes.byref(self.desc), K, len(N_list), _n_array(N_list), r, GROUP,
                                            c_void_p(self._base.data_ptr()), nbytes, c_void_p(_stream(stream))),
               "slim_grouped_layer_init")
        self.K, self.N, self.r = K, sum(N_list), r
        self.N_list = N_list

    @property
    def ref(self):
        return ctypes.byref(self.desc)

    def _view(self, addr: int, nbytes: int) -> torch.Tensor:
        off = addr - self._base.data_ptr()
        return self._base[off:off + nbytes]

    def canonical(self):
        """(vals [N][K/4] u8, meta [N][K/8] u8, scales [N][K/128] int16 bits) device views."""
        K, N = self.K, self.N
        vals = self._view(self.desc.vals, N * K // 4).view(N, K // 4)
        meta = self._view(self.desc.meta, N * K // 8).view(N, K // 8)
        sc = self._view(self.desc.scales, N * (K // GROUP) * 2).view(torch.int16).view(N, K // GROUP)
        return vals, meta, sc

    def regions(self) -> dict:
        """Device views of every byte the packer defines (alignment gaps excluded)."""
        K, N, d = self.K, self.N, self.desc
        r16 = d.r16
        out = {"vals": self._view(d.vals, N * K // 4), "meta": self._view(d.meta, N * K // 8),
               "scales": self._view(d.scales, N * (K // GROUP) * 2),
               "dec": self._view(d.dec, d.n_row_tiles * d.n_kblocks * 1600)}
        if self.r:
            out["Lf"] = self._view(d.Lf, d.rl16 * K * 2)
            out["Rf"] = self._view(d.Rf, d.n_row_tiles * 16 * r16 * 2)
            out["Rp"] = self._view(d.Rp, ((self.N + 511) // 512) * 512 * ((r16 + 63) // 64) * 64 * 2)
            out["Lp"] = self._view(d.Lp, K * d.rl16 * 2)
            if d.adapter_bits == 4:
                rq_tile = r16 // 16 * 128 + (self.r + 127) // 128 * 32
                out["Lq"] = self._view(d.Lq, d.rl16 // 16 * (K // GROUP) * 1056)
                out["Rq"] = self._view(d.Rq, d.n_row_tiles * rq_tile)
        return out

    @property
    def adapter_bits(self) -> int:
        return int(self.desc.adapter_bits)

    def set_adapter_bits(self, bits: int) -> None:
        """How the next pack stores the adapter: 16 (bf16) or 4 (quantized)."""
        _check(_lib.slim_layer_set_adapter_bits(self.ref, bits), "slim_layer_set_adapter_bits")

    def workspace_bytes(self, M: int) -> int:
        return int(_lib.slim_workspace_bytes(self.ref, M))

    def launches(self, M: int) -> int:
        """Kernels one linear() call launches for M tokens."""
        return int(_lib.slim_linear_launches(self.ref, M))

    def host_workspace_bytes(self, M: int) -> int:
        return int(_lib.slim_host_workspace_bytes(self.ref, M))


def pack(W: torch.Tensor, L: torch.Tensor | None = None, R: torch.Tensor | None = None, stream=None,
         check: bool = True, adapter_bits: int = 16) -> PackedLayer:
    """Quantize, 2:4-prune and pack W [N][K] (bf16, CUDA); copy in L [K][r], R [r][N]
    (adapter_bits=16), or quantize them to 4 bits as well (adapter_bits=4, see
    slim_layer_set_adapter_bits)."""
    N, K = W.shape
    r = 0 if L is None else L.shape[1]
    W = _as_bits(W, (N, K), "W")
    if r:
        L = _as_bits(L, (K, r), "L")
        R = _as_bits(R, (r, N), "R")
    layer = PackedLayer(K, N, r, W.device, stream)
    layer.set_adapter_bits(adapter_bits)
    _check(_lib.slim_pack(layer.ref, _ptr(W), _ptr(L) if r else None, _ptr(R) if r else None,
                          c_void_p(_stream(stream))), "slim_pack")
    if check:
        sync_status(layer, stream)
    return layer


def pack_grouped(Ws, Ls=None, Rs=None, stream=None, check: bool = True, adapter_bits: int = 16) -> PackedLayer:
    """Pack G linears that read the same X into one layer: W_g [N_g][K],
    L_g [K][r], R_g [r][N_g] (bf16, CUDA; all L_g / R_g None when r == 0).
    One linear() call then returns the G outputs side by side, [M][sum N_g]."""
    Ws = list(Ws)
    K = Ws[0].shape[1]
    N_list = [w.shape[0] for w in Ws]
    r = 0 if Ls is None else Ls[0].shape[1]
    W = torch.cat([_as_bits(w, (n, K), "W") for w, n in zip(Ws, N_list)], 0).contiguous()
    L = R = None
    if r:
        L = torch.cat([_as_bits(l, (K, r), "L") for l in Ls], 1).contiguous()
        R = torch.cat([_as_bits(rr, (r, n), "R") for rr, n in zip(Rs, N_list)], 1).contiguous()
    layer = PackedLayer(K, N_list, r, W.device, stream)
    layer.set_adapter_bits(adapter_bits)
    _check(_lib.slim_pack(layer.ref, _ptr(W), _ptr(L), _ptr(R), c_void_p(_stream(stream))), "slim_pack")
    if check:
        sync_status(layer, stream)
    return layer


def _zeros_on(nbytes: int, device, stream=None) -> torch.Tensor:
    """A zero-filled byte buffer whose allocation and fill are ordered on
    `stream` (torch's current stream when None), the stream the call that
    uses it runs on: a fill enqueued on another stream could still be
    running while the kernels read the buffer."""
    if stream is None:
        return torch.zeros(nbytes, dtype=torch.uint8, device=device)
    s = stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.ExternalStream(int(stream), device=device)
    with torch.cuda.stream(s):
        return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def workspace(layer: PackedLayer, M: int, device=None, stream=None) -> torch.Tensor | None:
    n = layer.workspace_bytes(M)
    if n == 0:
        return None
    # zero-filled: the forward's control words must start at zero
    return _zeros_on(n, device or layer.buf.device, stream)


def linear(layer: PackedLayer, X: torch.Tensor, Y: torch.Tensor | None = None,
           ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = X W_eff^T + (X L) R; X [M][K] bf16 CUDA -> Y [M][N] bf16."""
    M = X.shape[0]
    X = _as_bits(X, (M, layer.K), "X")
    if Y is None:
        Y = torch.empty(M, layer.N, dtype=torch.bfloat16, device=X.device)
    need = layer.workspace_bytes(M)
    if ws is None and need:
        ws = workspace(layer, M, X.device, stream)
    _check(_lib.slim_linear(layer.ref, _ptr(X), M, _ptr(Y), _ptr(ws), 0 if ws is None else ws.numel(),
                            c_void_p(_stream(stream))), "slim_linear")
    return Y


NOALLOC_SCRATCH_BYTES = 256 * 1024


def linear_noalloc(layer: PackedLayer, X: torch.Tensor, Y: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """Forward for callers that cannot allocate device memory: the adapter's
    X L scratch lives in a fixed array inside the library (NOALLOC_SCRATCH_BYTES
    per GPU), so no workspace is passed.  Calls that overlap on the GPU race on
    that array."""
    M = X.shape[0]
    X = _as_bits(X, (M, layer.K), "X")
    if Y is None:
        Y = torch.empty(M, layer.N, dtype=torch.bfloat16, device=X.device)
    _check(_lib.slim_linear_noalloc(layer.ref, _ptr(X), M, _ptr(Y), c_void_p(_stream(stream))),
           "slim_linear_noalloc")
    return Y


def linear_host(layer: PackedLayer, X_host: torch.Tensor, Y_host: torch.Tensor | None = None,
                ws: torch.Tensor | None = None, stream=None, wait: bool = True) -> torch.Tensor:
    """Forward on host tensors (pinned for speed); copies in and out.  With
    wait=False the copies and the forward are only enqueued on the stream:
    Y_host is valid once the stream has passed them."""
    M = X_host.shape[0]
    if X_host.is_cuda or tuple(X_host.shape) != (M, layer.K):
        raise ValueError("X_host must be a CPU tensor of shape [M][K]")
    X_host = X_host.contiguous()
    if Y_host is None:
        Y_host = torch.empty(M, layer.N, dtype=torch.bfloat16, pin_memory=True)
    if ws is None:
        ws = _zeros_on(layer.host_workspace_bytes(M), layer.buf.device, stream)
    fn = _lib.slim_linear_host if wait else _lib.slim_linear_host_async
    _check(fn(layer.ref, _ptr(X_host), M, _ptr(Y_host), _ptr(ws), ws.numel(), c_void_p(_stream(stream))),
           "slim_linear_host" if wait else "slim_linear_host_async")
    return Y_host


def test_wait_timeout(layer: PackedLayer, wait_us: int = 2000, stream=None) -> None:
    """Test aid: a device wait that nothing satisfies gives up after about
    wait_us and leaves SLIM_ERR_TIMEOUT in the layer's status word."""
    _check(_lib.slim_test_wait_timeout(layer.ref, int(wait_us), c_void_p(_stream(stream))), "slim_test_wait_timeout")


def test_stream_timeout(layer: PackedLayer, X: torch.Tensor, ws: torch.Tensor, wait_us: int = 2000,
                        Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Test aid: the single-launch decode kernel with waits for adapter
    partials that nothing writes; every output is stored as zeros and
    SLIM_ERR_TIMEOUT is left in the layer's status word."""
    M = X.shape[0]
    X = _as_bits(X, (M, layer.K), "X")
    if Y is None:
        Y = torch.empty(M, layer.N, dtype=torch.bfloat16, device=X.device)
    _check(_lib.slim_test_stream_timeout(layer.ref, _ptr(X), M, _ptr(Y), _ptr(ws), ws.numel(), int(wait_us),
                                         c_void_p(_stream(stream))), "slim_test_stream_timeout")
    return Y


def tuning_reload() -> None:
    """Re-read the SLIM_* tuning variables (the library reads them once, at its first call)."""
    _lib.slim_tuning_reload()


def unpack_dec(layer: PackedLayer, stream=None):
    """Dense int8 q [N][K] and fp16-bit scales [N][K/128] read back from the decode stream."""
    q = torch.empty(layer.N, layer.K, dtype=torch.int8, device=layer.buf.device)
    sc = torch.empty(layer.N, layer.K // GROUP, dtype=torch.int16, device=layer.buf.device)
    _check(_lib.slim_unpack_dec(layer.ref, _ptr(q), _ptr(sc), c_void_p(_stream(stream))), "slim_unpack_dec")
    return q, sc


def unpack_adapters(layer: PackedLayer, stream=None):
    """Expand a 4-bit adapter back to (q_L int8 [K][G r], s_L fp16 bits
    [K/128][G r], q_R int8 [r][N], s_R fp16 bits [ceil(r/128)][N]) device tensors."""
    dev = layer.buf.device
    Gr = layer.desc.n_groups * layer.r
    ngr = (layer.r + GROUP - 1) // GROUP
    qL = torch.empty(layer.K, Gr, dtype=torch.int8, device=dev)
    sL = torch.empty(layer.K // GROUP, Gr, dtype=torch.int16, device=dev)
    qR = torch.empty(layer.r, layer.N, dtype=torch.int8, device=dev)
    sR = torch.empty(ngr, layer.N, dtype=torch.int16, device=dev)
    _check(_lib.slim_unpack_adapters(layer.ref, _ptr(qL), _ptr(sL), _ptr(qR), _ptr(sR), c_void_p(_stream(stream))),
           "slim_unpack_adapters")
    return qL, sL, qR, sR


def sync_status(layer: PackedLayer, stream=None) -> None:
    _check(_lib.slim_sync_status(layer.ref, c_void_p(_stream(stream))), "device status")


def status_string(code: int) -> str:
    return _lib.slim_status_string(code).decode()


def abi_version() -> int:
    return int(_lib.slim_abi_version())
