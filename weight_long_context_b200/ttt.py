"""Thin Python binding of libttt (ctypes).  Argument marshalling only: every
step of the inner loop runs in the library's CUDA kernels.

The C names are re-exported one to one (ttt_create, ttt_prefill, ...); the
Handle class wraps them for torch tensors.  PyTorch provides device memory
and streams; nothing here computes any part of the method.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libttt.so")

TTT_OK = 0
STATUS_NAMES = ["TTT_OK", "TTT_ERR_INVALID_ARG", "TTT_ERR_SHAPE", "TTT_ERR_UNSUPPORTED",
                "TTT_ERR_WORKSPACE", "TTT_ERR_TOKEN_RANGE", "TTT_ERR_NONFINITE",
                "TTT_ERR_TIMEOUT", "TTT_ERR_CUDA"]
MLP = {"gelu": 0, "swiglu": 1}
PRECISION = {"fp32": 0, "bf16": 1}
REDUCTION = {"mean": 0, "sum": 1}
RULE = {"e2ttt": 0, "lact": 1}
HEAD = {"lm": 0, "recon": 1}

EXPORTED = ["ttt_create", "ttt_destroy", "ttt_workspace_size", "ttt_prefill", "ttt_prefill_noalloc",
            "ttt_prefill_host", "ttt_host_buffer_size",
            "ttt_prefill_profiled", "ttt_prefill_recon", "ttt_predict", "ttt_set_attention",
            "ttt_scalar_kernels", "ttt_scalar_heads", "ttt_gemm_bf16",
            "ttt_get_device_status", "ttt_selftest_bounded_wait", "ttt_status_string",
            "ttt_last_error"]


class TTTError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str = ""):
        name = STATUS_NAMES[code] if 0 <= code < len(STATUS_NAMES) else str(code)
        super().__init__(f"{where}: {name}" + (f" ({detail})" if detail else ""))
        self.code = code


class ttt_config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("hidden", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("n_blocks", ctypes.c_int32), ("mlp", ctypes.c_int32), ("has_static", ctypes.c_int32),
                ("precision", ctypes.c_int32), ("loss_reduction", ctypes.c_int32),
                ("rms_eps", ctypes.c_float), ("update_rule", ctypes.c_int32), ("head", ctypes.c_int32)]


class ttt_kernel_stat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 24), ("launches", ctypes.c_int64), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libttt.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libttt.so not found at {path}; run python -m weight_long_context_b200.build")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.ttt_create.argtypes = [ctypes.POINTER(ttt_config), P, P, P, ctypes.POINTER(P)]
    lib.ttt_create.restype = I32
    lib.ttt_destroy.argtypes = [P]
    lib.ttt_destroy.restype = None
    lib.ttt_workspace_size.argtypes = [P, I32, I32, I32, ctypes.POINTER(SZ)]
    lib.ttt_workspace_size.restype = I32
    lib.ttt_prefill.argtypes = [P, I32, I32, I32, P, P, P, P, P, P, P, P, P, SZ, P]
    lib.ttt_prefill.restype = I32
    lib.ttt_prefill_noalloc.argtypes = [P, I32, I32, I32, P, P, P, P, P, P, P, P, P]
    lib.ttt_host_buffer_size.argtypes = [P, I32, I32, I32, I32, ctypes.POINTER(SZ)]
    lib.ttt_host_buffer_size.restype = I32
    lib.ttt_prefill_host.argtypes = [P, I32, I32, I32, I32, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
    lib.ttt_prefill_host.restype = I32
    lib.ttt_prefill_recon.argtypes = [P, I32, I32, I32, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
    lib.ttt_prefill_recon.restype = I32
    lib.ttt_predict.argtypes = [P, I32, I32, I32, P, P, P, P, P, P, SZ, P]
    lib.ttt_predict.restype = I32
    lib.ttt_set_attention.argtypes = [P, I32, I32, P, P, P, ctypes.c_float]
    lib.ttt_set_attention.restype = I32
    lib.ttt_prefill_noalloc.restype = I32
    lib.ttt_prefill_profiled.argtypes = [P, I32, I32, I32, P, P, P, P, P, P, P, P, P, SZ, P,
                                         ctypes.POINTER(ttt_kernel_stat), I32, ctypes.POINTER(I32)]
    lib.ttt_prefill_profiled.restype = I32
    lib.ttt_scalar_kernels.argtypes = [I32, I32, I32, I32, P, P, P, P, P, P, P]
    F = ctypes.c_float
    lib.ttt_scalar_heads.argtypes = [I32, I32, I32, P, P, F, F, F, F, F, F, P, P, P, P]
    lib.ttt_scalar_heads.restype = I32
    lib.ttt_scalar_kernels.restype = I32
    I64 = ctypes.c_int64
    lib.ttt_gemm_bf16.argtypes = [I32, I32, I32, I32, P, I64, I64, I32, P, I64, I64, I32, P, I64, I64, P, SZ, P]
    lib.ttt_gemm_bf16.restype = I32
    lib.ttt_get_device_status.argtypes = [P, P]
    lib.ttt_get_device_status.restype = I32
    lib.ttt_selftest_bounded_wait.argtypes = [P, ctypes.c_uint32, P]
    lib.ttt_selftest_bounded_wait.restype = I32
    lib.ttt_status_string.argtypes = [I32]
    lib.ttt_status_string.restype = ctypes.c_char_p
    lib.ttt_last_error.argtypes = []
    lib.ttt_last_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(code: int, where: str):
    if code != TTT_OK:
        detail = load_library().ttt_last_error().decode(errors="replace")
        raise TTTError(code, where, detail)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> Optional[ctypes.c_void_p]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, dtype, name: str, device) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on the CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# --- the C names, re-exported --------------------------------------------------

def ttt_create(cfg: ttt_config, lm_head, rms_gain, static_w):
    lib = load_library()
    h = ctypes.c_void_p()
    _check(lib.ttt_create(ctypes.byref(cfg), _ptr(lm_head), _ptr(rms_gain), _ptr(static_w),
                          ctypes.byref(h)), "ttt_create")
    return h


def ttt_destroy(h):
    load_library().ttt_destroy(h)


def ttt_workspace_size(h, batch: int, T: int, b: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().ttt_workspace_size(h, batch, T, b, ctypes.byref(n)), "ttt_workspace_size")
    return n.value


def ttt_scalar_kernels(eta: torch.Tensor, beta: torch.Tensor, gamma: torch.Tensor, b: int, stream=None,
                       rule: str = "e2ttt"):
    """K1 alone: returns (KW [B,T], KM [B,T], consts [B,T/b,4]) as new CUDA tensors."""
    B, T = eta.shape
    for t, nm in ((eta, "eta"), (beta, "beta"), (gamma, "gamma")):
        _dev(t, torch.float32, nm, eta.device)
    KW = torch.empty_like(eta)
    KM = torch.empty_like(eta)
    consts = torch.empty((B, T // b if b > 0 else 0, 4), dtype=torch.float32, device=eta.device)
    _check(load_library().ttt_scalar_kernels(RULE[rule], B, T, b, _ptr(eta), _ptr(beta), _ptr(gamma), _ptr(KW),
                                             _ptr(KM), _ptr(consts), _stream_ptr(stream)),
           "ttt_scalar_kernels")
    return KW, KM, consts


def ttt_scalar_heads(hidden: torch.Tensor, heads: torch.Tensor, bias, eta_base: float, alpha_base: float,
                     tau: float, stream=None):
    """Input-dependent (eta, beta, gamma) [B, T] from hidden [B, T, d] and the
    heads [3, d] (w_eta, w_beta, w_alpha) with biases bias[0..2], as new CUDA tensors."""
    B, T, d = hidden.shape
    _dev(hidden, torch.float32, "hidden", hidden.device)
    _dev(heads, torch.float32, "heads", hidden.device)
    if tuple(heads.shape) != (3, d):
        raise ValueError("heads must be [3, d]")
    eta = torch.empty((B, T), dtype=torch.float32, device=hidden.device)
    beta = torch.empty_like(eta)
    gamma = torch.empty_like(eta)
    _check(load_library().ttt_scalar_heads(B, T, d, _ptr(hidden), _ptr(heads), float(bias[0]), float(bias[1]),
                                           float(bias[2]), eta_base, alpha_base, tau, _ptr(eta), _ptr(beta),
                                           _ptr(gamma), _stream_ptr(stream)), "ttt_scalar_heads")
    return eta, beta, gamma


def ttt_gemm_bf16(A: torch.Tensor, B: torch.Tensor, a_kmajor: bool = True, b_kmajor: bool = True,
                  out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """D[z] = A[z] B[z]^T on the tcgen05 engine.  A, B: bf16 CUDA tensors of shape
    [batch, M, K] / [batch, N, K] when K-major, [batch, K, M] / [batch, K, N] when
    MN-major (2-D inputs are batch 1).  Returns fp32 [batch, M, N]."""
    A3 = A if A.dim() == 3 else A.unsqueeze(0)
    B3 = B if B.dim() == 3 else B.unsqueeze(0)
    _dev(A3, torch.bfloat16, "A", A.device)
    _dev(B3, torch.bfloat16, "B", A.device)
    batch = A3.shape[0]
    M, K = (A3.shape[1], A3.shape[2]) if a_kmajor else (A3.shape[2], A3.shape[1])
    N = B3.shape[1] if b_kmajor else B3.shape[2]
    if out is None:
        out = torch.empty((batch, M, N), dtype=torch.float32, device=A.device)
    sA = A3.shape[1] * A3.shape[2] if batch > 1 else 0
    sB = B3.shape[1] * B3.shape[2] if batch > 1 else 0
    _check(load_library().ttt_gemm_bf16(M, N, K, batch, _ptr(A3), A3.shape[2], sA, int(a_kmajor), _ptr(B3),
                                        B3.shape[2], sB, int(b_kmajor), _ptr(out), N, M * N,
                                        _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                        _stream_ptr(stream)), "ttt_gemm_bf16")
    return out if A.dim() == 3 else out[0]


def ttt_status_string(code: int) -> str:
    return load_library().ttt_status_string(code).decode()


def ttt_last_error() -> str:
    return load_library().ttt_last_error().decode(errors="replace")


# --- object wrapper ------------------------------------------------------------

class Handle:
    """A libttt handle with the frozen head / static weights bound.

    lm_head [V, d], rms_gain [d], static_w [n_blocks*m*h*d] or None: float32
    tensors on the CUDA device (copied by the library).
    """

    def __init__(self, d: int, hidden: int, vocab: int, n_blocks: int, mlp: str, has_static: bool,
                 precision: str, lm_head: torch.Tensor, rms_gain: torch.Tensor,
                 static_w: Optional[torch.Tensor] = None, rms_eps: float = 1e-6,
                 reduction: str = "mean", update_rule: str = "e2ttt", head: str = "lm",
                 device: Optional[torch.device] = None):
        dev = lm_head.device if lm_head is not None else device
        if dev is None:
            raise ValueError("device is required when lm_head is None")
        if head == "lm":
            _dev(lm_head, torch.float32, "lm_head", dev)
            _dev(rms_gain, torch.float32, "rms_gain", dev)
        if static_w is not None:
            _dev(static_w, torch.float32, "static_w", dev)
        self.cfg = ttt_config(d, hidden, vocab, n_blocks, MLP[mlp], int(bool(has_static)),
                              PRECISION[precision], REDUCTION[reduction], rms_eps, RULE[update_rule], HEAD[head])
        self.device = dev
        self.n_mats = 2 if mlp == "gelu" else 3
        with torch.cuda.device(dev):
            self._h = ttt_create(self.cfg, lm_head, rms_gain, static_w)
        self._ws = None
        self._hbuf = None   # device buffer of the host-buffer prefill, grown on demand

    def set_attention(self, n_heads: int, window: int, attn_w, ln_gain, ln_bias, ln_eps: float = 1e-5):
        """Frozen sliding-window attention in front of every updated block:
        attn_w [n_blocks, 4, d, d] (Wq, Wk, Wv, Wo), ln_gain / ln_bias
        [n_blocks, d], float32 CUDA tensors (copied).  n_heads = 0 removes it."""
        if n_heads:
            for t, nm in ((attn_w, "attn_w"), (ln_gain, "ln_gain"), (ln_bias, "ln_bias")):
                _dev(t, torch.float32, nm, self.device)
            L, d = self.cfg.n_blocks, self.cfg.d
            if attn_w.numel() != L * 4 * d * d or ln_gain.numel() != L * d or ln_bias.numel() != L * d:
                raise ValueError("attn_w must be [n_blocks, 4, d, d], ln_gain and ln_bias [n_blocks, d]")
        with torch.cuda.device(self.device):
            _check(load_library().ttt_set_attention(self._h, n_heads, window, _ptr(attn_w), _ptr(ln_gain),
                                                    _ptr(ln_bias), ln_eps), "ttt_set_attention")
        self._ws = None
        self._hbuf = None

    # workspace cached per handle, grown on demand
    def workspace(self, batch: int, T: int, b: int) -> torch.Tensor:
        need = ttt_workspace_size(self._h, batch, T, b)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def prefill(self, hidden, tokens, W, M, eta, beta, gamma, b: int,
                chunk_loss: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Run the inner loop on device tensors.  W and M are updated in place.

        hidden [B,T,d] f32, tokens [B,T] i32, W/M [B*n_blocks*m*h*d] f32,
        eta/beta/gamma [B,T] f32.  Returns chunk_loss [B, T/b] (f32, device).
        """
        dev = self.device
        B, T, d = hidden.shape
        for t, nm in ((hidden, "hidden"), (W, "W"), (M, "M"), (eta, "eta"), (beta, "beta"),
                      (gamma, "gamma")):
            _dev(t, torch.float32, nm, dev)
        _dev(tokens, torch.int32, "tokens", dev)
        nparams = B * self.cfg.n_blocks * self.n_mats * self.cfg.hidden * self.cfg.d
        if W.numel() != nparams or M.numel() != nparams:
            raise ValueError(f"W and M must hold {nparams} floats")
        if tuple(tokens.shape) != (B, T) or tuple(eta.shape) != (B, T):
            raise ValueError("tokens / eta / beta / gamma must be [B, T]")
        nc = T // b if b > 0 else 0
        if chunk_loss is None:
            chunk_loss = torch.empty((B, nc), dtype=torch.float32, device=dev)
        ws = self.workspace(B, T, b)
        _check(load_library().ttt_prefill(self._h, B, T, b, _ptr(hidden), _ptr(tokens), _ptr(W), _ptr(M),
                                          _ptr(eta), _ptr(beta), _ptr(gamma), _ptr(chunk_loss),
                                          _ptr(ws), ws.numel(), _stream_ptr(stream)), "ttt_prefill")
        return chunk_loss

    def predict(self, hidden, tokens, W, b: int, token_loss: bool = False,
                group_loss: Optional[torch.Tensor] = None, stream=None):
        """Final prediction at fixed fast weights W (no update) on device tensors:
        hidden [B,T,d] f32, tokens [B,T] i32, W [B*n_blocks*m*h*d] f32.  b rows
        per sequence per pass (any divisor of T).  Returns (group_loss [B, T/b],
        token_loss [B, T] or None) on the device."""
        dev = self.device
        B, T, d = hidden.shape
        _dev(hidden, torch.float32, "hidden", dev)
        _dev(W, torch.float32, "W", dev)
        _dev(tokens, torch.int32, "tokens", dev)
        nparams = B * self.cfg.n_blocks * self.n_mats * self.cfg.hidden * self.cfg.d
        if W.numel() != nparams:
            raise ValueError(f"W must hold {nparams} floats")
        if tuple(tokens.shape) != (B, T):
            raise ValueError("tokens must be [B, T]")
        nc = T // b if b > 0 else 0
        if group_loss is None:
            group_loss = torch.empty((B, nc), dtype=torch.float32, device=dev)
        tl = torch.empty((B, T), dtype=torch.float32, device=dev) if token_loss else None
        ws = self.workspace(B, T, b)
        _check(load_library().ttt_predict(self._h, B, T, b, _ptr(hidden), _ptr(tokens), _ptr(W),
                                          _ptr(group_loss), _ptr(tl), _ptr(ws), ws.numel(), _stream_ptr(stream)),
               "ttt_predict")
        return group_loss, tl

    def predict_host(self, hidden, tokens, W, b: int, stream=None):
        """End-to-end final prediction on HOST tensors: copies hidden, tokens and
        W in, runs, copies the group losses back.  Returns group_loss [B, T/b]
        (host)."""
        dev = self.device
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        with torch.cuda.stream(st):
            d_in = [t.to(dev, non_blocking=True) for t in (hidden, tokens, W)]
            grp, _ = self.predict(*d_in, b=b, stream=st)
            out = torch.empty(grp.shape, dtype=grp.dtype, pin_memory=True)
            out.copy_(grp, non_blocking=True)
        st.synchronize()
        return out

    def prefill_recon(self, K, V, Q, W, M, eta, beta, gamma, b: int, O: Optional[torch.Tensor] = None,
                      chunk_loss: Optional[torch.Tensor] = None, stream=None):
        """E2-TTT's own layer on device tensors (handle created with head="recon"):
        K, V, Q [B,T,d] f32; W/M [B*m*h*d] f32 updated in place; eta/beta/gamma
        [B,T].  Returns (chunk_loss [B, T/b], O [B,T,d]) on the device."""
        dev = self.device
        B, T, d = K.shape
        for t, nm in ((K, "K"), (V, "V"), (Q, "Q"), (W, "W"), (M, "M"), (eta, "eta"), (beta, "beta"),
                      (gamma, "gamma")):
            _dev(t, torch.float32, nm, dev)
        if tuple(V.shape) != (B, T, d) or tuple(Q.shape) != (B, T, d):
            raise ValueError("K, V and Q must have the same shape [B, T, d]")
        nparams = B * self.n_mats * self.cfg.hidden * self.cfg.d
        if W.numel() != nparams or M.numel() != nparams:
            raise ValueError(f"W and M must hold {nparams} floats")
        nc = T // b if b > 0 else 0
        if chunk_loss is None:
            chunk_loss = torch.empty((B, nc), dtype=torch.float32, device=dev)
        if O is None:
            O = torch.empty((B, T, d), dtype=torch.float32, device=dev)
        ws = self.workspace(B, T, b)
        _check(load_library().ttt_prefill_recon(self._h, B, T, b, _ptr(K), _ptr(V), _ptr(Q), _ptr(W), _ptr(M),
                                                _ptr(eta), _ptr(beta), _ptr(gamma), _ptr(O), _ptr(chunk_loss),
                                                _ptr(ws), ws.numel(), _stream_ptr(stream)), "ttt_prefill_recon")
        return chunk_loss, O

    def prefill_recon_host(self, K, V, Q, W0, M0, eta, beta, gamma, b: int, stream=None):
        """End-to-end reconstruction call on HOST tensors: copies in, runs, copies
        W, M, the chunk losses and the outputs back.  Returns host tensors
        (W, M, chunk_loss, O)."""
        dev = self.device
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        with torch.cuda.stream(st):
            d_in = [t.to(dev, non_blocking=True) for t in (K, V, Q, W0, M0, eta, beta, gamma)]
            loss, O = self.prefill_recon(*d_in, b=b, stream=st)
            outs = []
            for t in (d_in[3], d_in[4], loss, O):
                o = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                o.copy_(t, non_blocking=True)
                outs.append(o)
        st.synchronize()
        return tuple(outs)

    def prefill_profiled(self, hidden, tokens, W, M, eta, beta, gamma, b: int, stream=None):
        """ttt_prefill_profiled: same results as prefill (W, M updated in place),
        plus per-kernel-class stats.  Returns (chunk_loss, [dict, ...])."""
        B, T, d = hidden.shape
        nc = T // b if b > 0 else 0
        loss = torch.empty((B, nc), dtype=torch.float32, device=self.device)
        ws = self.workspace(B, T, b)
        stats = (ttt_kernel_stat * 32)()
        n = ctypes.c_int32()
        _check(load_library().ttt_prefill_profiled(self._h, B, T, b, _ptr(hidden), _ptr(tokens), _ptr(W), _ptr(M),
                                                   _ptr(eta), _ptr(beta), _ptr(gamma), _ptr(loss), _ptr(ws),
                                                   ws.numel(), _stream_ptr(stream), stats, 32, ctypes.byref(n)),
               "ttt_prefill_profiled")
        out = [dict(name=stats[i].name.decode(), launches=stats[i].launches, ms=stats[i].ms,
                    flops=stats[i].flops, bytes=stats[i].bytes) for i in range(n.value)]
        return loss, out

    def prefill_host(self, hidden, tokens, W0, M0, eta, beta, gamma, b: int, stream=None, scalar_heads=None,
                     seg_chunks: int = 0):
        """End-to-end call on HOST tensors: the inputs go to the device, the
        inner loop runs, W, M and the chunk losses come back.  Returns
        (W, M, chunk_loss) as new host tensors (pinned).  Without scalar heads
        this is ttt_prefill_host (the sequence streamed in segments of
        seg_chunks chunks, copies overlapping the compute; pass pinned host
        tensors).  scalar_heads = (heads [3, d] CUDA tensor, bias[3],
        eta_base, alpha_base, tau): the scalars come from ttt_scalar_heads on
        the device (eta, beta, gamma are then ignored), after a plain copy of
        the inputs."""
        dev = self.device
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        if scalar_heads is not None:
            with torch.cuda.stream(st):
                d_in = [t.to(dev, non_blocking=True) for t in (hidden, tokens, W0, M0)]
                d_in += list(ttt_scalar_heads(d_in[0], *scalar_heads, stream=st))
                loss = self.prefill(*d_in, b=b, stream=st)
                outs = []
                for t in (d_in[2], d_in[3], loss):
                    o = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                    o.copy_(t, non_blocking=True)
                    outs.append(o)
            st.synchronize()
            return tuple(outs)
        for name, t, dt in (("hidden", hidden, torch.float32), ("tokens", tokens, torch.int32),
                            ("W0", W0, torch.float32), ("M0", M0, torch.float32), ("eta", eta, torch.float32),
                            ("beta", beta, torch.float32), ("gamma", gamma, torch.float32)):
            if t.device.type != "cpu" or t.dtype != dt or not t.is_contiguous():
                raise ValueError(f"{name}: expected a contiguous {dt} host tensor")
        B, T = hidden.shape[0], hidden.shape[1]
        lib = load_library()
        need = ctypes.c_size_t(0)
        _check(lib.ttt_host_buffer_size(self._h, B, T, b, seg_chunks, ctypes.byref(need)), "ttt_host_buffer_size")
        if self._hbuf is None or self._hbuf.numel() < need.value:
            self._hbuf = torch.empty(need.value, dtype=torch.uint8, device=dev)
        W = torch.empty(W0.shape, dtype=torch.float32, pin_memory=True)
        M = torch.empty(M0.shape, dtype=torch.float32, pin_memory=True)
        loss = torch.empty((B, T // b if b > 0 else 0), dtype=torch.float32, pin_memory=True)
        with torch.cuda.device(dev):
            _check(lib.ttt_prefill_host(self._h, B, T, b, seg_chunks, _ptr(hidden), _ptr(tokens), _ptr(W0),
                                        _ptr(M0), _ptr(W), _ptr(M), _ptr(eta), _ptr(beta), _ptr(gamma), _ptr(loss),
                                        _ptr(self._hbuf), self._hbuf.numel(), _stream_ptr(st)), "ttt_prefill_host")
        return W, M, loss

    def device_status(self, stream=None) -> int:
        return load_library().ttt_get_device_status(self._h, _stream_ptr(stream))

    def selftest_bounded_wait(self, spin_limit: int, stream=None):
        _check(load_library().ttt_selftest_bounded_wait(self._h, spin_limit, _stream_ptr(stream)),
               "ttt_selftest_bounded_wait")

    def close(self):
        if getattr(self, "_h", None):
            ttt_destroy(self._h)
            self._h = None
        self._ws = None
        self._hbuf = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
