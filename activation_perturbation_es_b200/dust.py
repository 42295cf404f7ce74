"""Python binding of libdust.so (the C ABI in include/dust.h).

Argument marshalling only: tensors must be CUDA tensors of the documented
dtype and layout; this module turns them into pointers and the current torch
stream, allocates the caller-owned outputs and workspace with torch, and calls
the library.  Every step of the estimator runs in the library's kernels; there
is no CPU or PyTorch fallback, and a missing library raises.

Names follow the C ABI with the ``dust_`` prefix dropped.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libdust.so")

F32, BF16 = 0, 1
STATUS = {0: "DUST_OK", 1: "DUST_ERR_INVALID_ARG", 2: "DUST_ERR_UNSUPPORTED", 3: "DUST_ERR_ALIGNMENT",
          4: "DUST_ERR_WORKSPACE", 5: "DUST_ERR_CUDA", 6: "DUST_ERR_TIMEOUT"}


class DustError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class _Noise(C.Structure):
    _fields_ = [("seed", C.c_uint32), ("layer", C.c_uint32), ("draw_begin", C.c_uint32),
                ("draw_count", C.c_uint32), ("K_total", C.c_uint32), ("sigma", C.c_float),
                ("token_begin", C.c_uint32)]


@dataclass(frozen=True)
class Noise:
    """Which draws of which layer a call handles, and the global index of its
    first token (dust_noise)."""
    seed: int
    layer: int
    draw_begin: int
    draw_count: int
    K_total: int
    sigma: float
    token_begin: int = 0

    def c(self) -> _Noise:
        return _Noise(self.seed, self.layer, self.draw_begin, self.draw_count, self.K_total, self.sigma,
                      self.token_begin)


_lib = None
_vp, _sz, _i, _f, _u = C.c_void_p, C.c_size_t, C.c_int, C.c_float, C.c_uint32

_SIGS = {
    "dust_status_string": ([_i], C.c_char_p),
    "dust_last_error": ([], C.c_char_p),
    "dust_abi_version": ([], _i),
    "dust_check_offsets": ([_vp, _i, _i], _i),
    "dust_poll_status": ([_vp, _vp], _i),
    "dust_selftest_bounded_wait": ([_vp, _u, _vp], _i),
    "dust_reward_scan": ([_vp, _vp, _i, _i, _vp, _i, _f, _vp], _i),
    "dust_reward_scan_split": ([_vp, _vp, _i, _i, _vp, _i, _f, _vp, _sz, _vp], _i),
    "dust_reward_scan_split_workspace": ([_i, _i], _sz),
    "dust_layer_estimate": ([_vp, _i, _i, _i, _vp, _i, _f, _Noise, _vp, _vp, _i, _vp, _sz, _vp], _i),
    "dust_layer_estimate_workspace": ([_i, _i, _i, _i, _f], _sz),
    "dust_layer_estimate_noalloc": ([_vp, _i, _i, _vp, _i, _f, _Noise, _vp, _vp, _i, _vp], _i),
    "dust_layer_estimate_weight_grad": ([_vp, _i, _i, _i, _vp, _i, _f, _Noise, _vp, _i, _vp, _i, _vp, _vp, _sz, _vp],
                                        _i),
    "dust_layer_estimate_weight_grad_workspace": ([_i, _i, _i, _i, _i, _f], _sz),
    "dust_weight_grad": ([_vp, _i, _vp, _i, _i, _i, _i, _vp, _i, _vp, _sz, _vp], _i),
    "dust_weight_grad_workspace": ([_i, _i, _i, _i, _i], _sz),
    "dust_logits": ([_vp, _vp, _i, _i, _i, _i, _vp, _vp, _sz, _vp], _i),
    "dust_logits_workspace": ([_i, _i, _i, _i], _sz),
    "dust_head_row_stats": ([_vp, _vp, _i, _i, _vp, _vp, _vp], _i),
    "dust_head_step": ([_vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _i, _Noise, _vp, _vp, _vp, _vp, _i, _vp, _sz,
                        _vp], _i),
    "dust_head_step_workspace": ([_i, _i, _i, _i, _i, _i, _i, _i], _sz),
    "dust_head_bp_grad": ([_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _sz, _vp], _i),
    "dust_head_bp_grad_workspace": ([_i, _i, _i, _i], _sz),
    "dust_cosine": ([_vp, _vp, C.c_longlong, _vp, _vp, _sz, _vp], _i),
    "dust_cosine_workspace": ([], _sz),
    "dust_noise_fill": ([_Noise, _u, _i, _i, _i, _i, _vp, _vp], _i),
    "dust_noise_sum": ([_Noise, _i, _i, _vp, _vp], _i),
    "dust_box_muller_words": ([_vp, _vp, C.c_longlong, _vp, _vp, _vp], _i),
    "dust_synth_costs": ([_vp, _i, _i, _Noise, _f, _vp, _vp], _i),
    "dust_toy_suffix_losses": ([_vp, _i, _i, _vp, _i, _vp, _vp, _vp, _vp, _i, _vp, _i, _vp, _Noise, _vp, _vp,
                                _vp, _sz, _vp], _i),
    "dust_toy_suffix_workspace": ([_i, _i, _i, _i, _i], _sz),
    "dust_attention_internal_costs": ([_vp, _i, _i, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _Noise, _vp,
                                       _vp, _sz, _vp], _i),
    "dust_attention_internal_costs_workspace": ([_i, _i, _i, _i], _sz),
}


def lib() -> C.CDLL:
    """Load libdust.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m activation_perturbation_es_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != 0:
        raise DustError(status, lib().dust_last_error().decode())


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _opt(t, name, dtype=None):
    return None if t is None else _dev(t, name, dtype)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


_ws = {}


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A cached caller-owned workspace of at least nbytes, one per (device,
    current stream): calls on one stream run in order and can share it, calls
    on different streams get different buffers.  Grows (reallocates) on
    demand, so warm a path up once before capturing it in a CUDA graph."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    key = (dev, torch.cuda.current_stream(dev).cuda_stream)
    cur = _ws.get(key)
    if cur is None or cur.numel() < nbytes:
        new = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
        if cur is not None:
            new[:256].copy_(cur[:256])     # keep a status word that earlier calls may have set
        cur = new
        _ws[key] = cur
    return cur


def check_offsets(seq_offsets, T: int) -> None:
    """Validate sequence offsets on the host (numpy / CPU tensor / list)."""
    off = np.ascontiguousarray(np.asarray(seq_offsets.cpu() if isinstance(seq_offsets, torch.Tensor)
                                          else seq_offsets), dtype=np.int32)
    _check(lib().dust_check_offsets(off.ctypes.data, len(off) - 1, T))


def poll_status(ws: torch.Tensor) -> None:
    _check(lib().dust_poll_status(_dev(ws, "ws"), _stream()))


def poll_all(device=None) -> str:
    """dust_poll_status on every cached workspace of `device` (default: the
    current one), each on the stream it serves.  Raises DustError with
    DUST_ERR_TIMEOUT when a kernel's bounded wait ran out since the last poll
    (the word is cleared); returns "ok" otherwise."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    failed = None
    for (d, stream), ws in list(_ws.items()):
        if d != dev:
            continue
        st = lib().dust_poll_status(ws.data_ptr(), stream)
        if st != 0 and failed is None:
            failed = DustError(st, lib().dust_last_error().decode())
    if failed is not None:
        raise failed
    return "ok"


def selftest_bounded_wait(ws: torch.Tensor, polls: int = 4096) -> None:
    _check(lib().dust_selftest_bounded_wait(_dev(ws, "ws"), polls, _stream()))


# ------------------------------------------------------------------ a4
def reward_scan(c: torch.Tensor, seq_offsets: torch.Tensor, gamma: float, out: torch.Tensor | None = None):
    K, T = c.shape
    r = torch.empty_like(c) if out is None else out
    _check(lib().dust_reward_scan(_dev(c, "c", torch.float32), _dev(r, "r", torch.float32), K, T,
                                  _dev(seq_offsets, "seq_offsets", torch.int32), seq_offsets.numel() - 1,
                                  float(gamma), _stream()))
    return r


def reward_scan_split(c: torch.Tensor, seq_offsets: torch.Tensor, gamma: float, out: torch.Tensor | None = None):
    """dust_reward_scan_split: the reward scan over 1024-token chunks (for few long sequences)."""
    K, T = c.shape
    r = torch.empty_like(c) if out is None else out
    ws = workspace(lib().dust_reward_scan_split_workspace(K, T), c.device)
    _check(lib().dust_reward_scan_split(_dev(c, "c", torch.float32), _dev(r, "r", torch.float32), K, T,
                                        _dev(seq_offsets, "seq_offsets", torch.int32), seq_offsets.numel() - 1,
                                        float(gamma), ws.data_ptr(), ws.numel(), _stream()))
    return r


# ------------------------------------------------------------------ a5
def layer_estimate(c_or_r: torch.Tensor, is_r: bool, seq_offsets, gamma: float, noise: Noise, d_out: int,
                   g_hat: torch.Tensor | None = None, g_hat_bf16: torch.Tensor | bool | None = None,
                   accumulate: bool = False):
    """Returns (g_hat [T][d_out] fp32, g_hat_bf16 or None)."""
    nd, T = c_or_r.shape
    if nd != noise.draw_count:
        raise ValueError("c_or_r must have draw_count rows")
    dev = c_or_r.device
    if g_hat is None:
        g_hat = torch.empty(T, d_out, dtype=torch.float32, device=dev)
    if g_hat_bf16 is True:
        g_hat_bf16 = torch.empty(T, d_out, dtype=torch.bfloat16, device=dev)
    elif g_hat_bf16 is False:
        g_hat_bf16 = None
    need = lib().dust_layer_estimate_workspace(nd, T, d_out, int(bool(is_r)), float(gamma))
    ws = workspace(need, dev)
    offs = None if seq_offsets is None else _dev(seq_offsets, "seq_offsets", torch.int32)
    n_seq = 1 if seq_offsets is None else seq_offsets.numel() - 1
    _check(lib().dust_layer_estimate(_dev(c_or_r, "c_or_r", torch.float32), int(bool(is_r)), T, d_out, offs, n_seq,
                                     float(gamma), noise.c(), _dev(g_hat, "g_hat", torch.float32),
                                     _opt(g_hat_bf16, "g_hat_bf16", torch.bfloat16), int(bool(accumulate)),
                                     ws.data_ptr(), ws.numel(), _stream()))
    return g_hat, g_hat_bf16


def layer_estimate_weight_grad(c_or_r: torch.Tensor, is_r: bool, seq_offsets, gamma: float, noise: Noise,
                               X: torch.Tensor, d_out: int, G_W: torch.Tensor | None = None, accumulate: bool = False,
                               g_hat: torch.Tensor | bool | None = None):
    """dust_layer_estimate_weight_grad: G_W [d_out][d_in] fp32 from costs or
    rewards and bf16 X [T][d_in] in one fused pass (g never leaves the chip).
    g_hat=True (or a tensor) also returns g. Returns (G_W, g_hat or None)."""
    nd, T = c_or_r.shape
    if nd != noise.draw_count:
        raise ValueError("c_or_r must have draw_count rows")
    if X.dim() != 2 or X.shape[0] != T:
        raise ValueError("X must be [T][d_in]")
    d_in = X.shape[1]
    dev = c_or_r.device
    if G_W is None:
        G_W = torch.empty(d_out, d_in, dtype=torch.float32, device=dev)
    if g_hat is True:
        g_hat = torch.empty(T, d_out, dtype=torch.float32, device=dev)
    elif g_hat is False:
        g_hat = None
    need = lib().dust_layer_estimate_weight_grad_workspace(nd, T, d_in, d_out, int(bool(is_r)), float(gamma))
    ws = workspace(need, dev)
    offs = None if seq_offsets is None else _dev(seq_offsets, "seq_offsets", torch.int32)
    n_seq = 1 if seq_offsets is None else seq_offsets.numel() - 1
    _check(lib().dust_layer_estimate_weight_grad(
        _dev(c_or_r, "c_or_r", torch.float32), int(bool(is_r)), T, d_out, offs, n_seq, float(gamma), noise.c(),
        _dev(X, "X", torch.bfloat16), d_in, _dev(G_W, "G_W", torch.float32), int(bool(accumulate)),
        _opt(g_hat, "g_hat", torch.float32), ws.data_ptr(), ws.numel(), _stream()))
    return G_W, g_hat


def layer_estimate_noalloc(c: torch.Tensor, seq_offsets, gamma: float, noise: Noise, d_out: int,
                           g_hat: torch.Tensor | None = None, g_hat_bf16: torch.Tensor | None = None,
                           accumulate: bool = False):
    """dust_layer_estimate_noalloc: the estimate from costs c with the library's
    static scratch instead of a workspace (for callers that cannot allocate).
    Returns (g_hat, g_hat_bf16 or None)."""
    nd, T = c.shape
    if nd != noise.draw_count:
        raise ValueError("c must have draw_count rows")
    if g_hat is None:
        g_hat = torch.empty(T, d_out, dtype=torch.float32, device=c.device)
    offs = None if seq_offsets is None else _dev(seq_offsets, "seq_offsets", torch.int32)
    n_seq = 1 if seq_offsets is None else seq_offsets.numel() - 1
    _check(lib().dust_layer_estimate_noalloc(_dev(c, "c", torch.float32), T, d_out, offs, n_seq, float(gamma),
                                             noise.c(), _dev(g_hat, "g_hat", torch.float32),
                                             _opt(g_hat_bf16, "g_hat_bf16", torch.bfloat16),
                                             int(bool(accumulate)), _stream()))
    return g_hat, g_hat_bf16


# ------------------------------------------------------------------ a6
def weight_grad(g_hat: torch.Tensor, X: torch.Tensor, G_W: torch.Tensor | None = None, accumulate: bool = False):
    """G_W [d_out][d_in] fp32 = g_hat^T X; g_hat and X each fp32 or bf16 (they may differ)."""
    T, d_out = g_hat.shape
    d_in = X.shape[1]
    if X.shape[0] != T:
        raise ValueError("g_hat and X must share T")
    g_dt, x_dt = _dtype_code(g_hat), _dtype_code(X)
    if G_W is None:
        G_W = torch.empty(d_out, d_in, dtype=torch.float32, device=X.device)
    ws = workspace(lib().dust_weight_grad_workspace(T, d_in, d_out, g_dt, x_dt), X.device)
    _check(lib().dust_weight_grad(_dev(g_hat, "g_hat"), g_dt, _dev(X, "X"), x_dt, T, d_in, d_out,
                                  _dev(G_W, "G_W", torch.float32), int(bool(accumulate)), ws.data_ptr(),
                                  ws.numel(), _stream()))
    return G_W


# ------------------------------------------------------------------ a2
def logits(X: torch.Tensor, W: torch.Tensor, Z: torch.Tensor | None = None):
    T, d_in = X.shape
    V = W.shape[0]
    dt = _dtype_code(X)
    if W.dtype != X.dtype or W.shape[1] != d_in:
        raise ValueError("X and W must share d_in and dtype")
    if Z is None:
        Z = torch.empty(T, V, dtype=torch.float32, device=X.device)
    ws = workspace(lib().dust_logits_workspace(T, d_in, V, dt), X.device)
    _check(lib().dust_logits(_dev(X, "X"), _dev(W, "W"), dt, T, d_in, V, _dev(Z, "Z", torch.float32),
                             ws.data_ptr(), ws.numel(), _stream()))
    return Z


def head_row_stats(Z: torch.Tensor, targets: torch.Tensor):
    T, V = Z.shape
    lse = torch.empty(T, dtype=torch.float32, device=Z.device)
    ell = torch.empty(T, dtype=torch.float32, device=Z.device)
    _check(lib().dust_head_row_stats(_dev(Z, "Z", torch.float32), _dev(targets, "targets", torch.int32), T, V,
                                     lse.data_ptr(), ell.data_ptr(), _stream()))
    return lse, ell


# ------------------------------------------------------------------ head step
def head_step(targets: torch.Tensor, Vc: int, noise: Noise, *, Z: torch.Tensor | None = None,
              X: torch.Tensor | None = None, W: torch.Tensor | None = None, V: int | None = None,
              want_c: bool = False, want_bf16: bool = False, want_G_W: bool = False,
              g_hat: torch.Tensor | None = None, g_hat_bf16: torch.Tensor | None = None,
              accumulate: bool = False, chunk_begin: int = 0, chunk_count: int | None = None):
    """Returns dict with g_hat, and c / g_hat_bf16 / G_W when requested.  The
    chunk range [chunk_begin, chunk_begin + chunk_count) (default: every chunk)
    sets the outputs' vocabulary columns / rows: g_hat [T][chunk_count Vc],
    c [chunk_count][draw_count][T], G_W [chunk_count Vc][d_in]."""
    T = targets.numel()
    dev = targets.device
    if Z is not None:
        V = Z.shape[1]
    elif W is not None:
        V = W.shape[0]
    if V is None:
        raise ValueError("need Z or W")
    if chunk_count is None:
        chunk_count = V // Vc - chunk_begin
    Vr = chunk_count * Vc
    ref = X if X is not None else W
    dt = _dtype_code(ref) if ref is not None else F32
    d_in = X.shape[1] if X is not None else (W.shape[1] if W is not None else 0)
    if g_hat is None:
        g_hat = torch.empty(T, Vr, dtype=torch.float32, device=dev)
    c = torch.empty(chunk_count, noise.draw_count, T, dtype=torch.float32, device=dev) if want_c else None
    g16 = g_hat_bf16
    if g16 is None and want_bf16:
        g16 = torch.empty(T, Vr, dtype=torch.bfloat16, device=dev)
    G_W = torch.empty(Vr, d_in, dtype=torch.float32, device=dev) if want_G_W else None
    need = lib().dust_head_step_workspace(T, d_in, V, Vc, chunk_count, dt, int(Z is not None), int(want_G_W))
    ws = workspace(need, dev)
    _check(lib().dust_head_step(_opt(X, "X"), _opt(W, "W"), dt, _opt(Z, "Z", torch.float32),
                                _dev(targets, "targets", torch.int32), T, d_in, V, Vc, chunk_begin, chunk_count,
                                noise.c(), _opt(c, "c"), _dev(g_hat, "g_hat", torch.float32), _opt(g16, "g_hat_bf16"),
                                _opt(G_W, "G_W"), int(bool(accumulate)), ws.data_ptr(), ws.numel(), _stream()))
    return {"g_hat": g_hat, "c": c, "g_hat_bf16": g16, "G_W": G_W}


# ------------------------------------------------------------------ cosine tuner
def head_bp_grad(Z: torch.Tensor, targets: torch.Tensor, X: torch.Tensor, G_bp: torch.Tensor | None = None):
    """Backprop gradient of the head's summed cross entropy, sum_t (softmax(z_t) - e_y) x_t^T."""
    T, V = Z.shape
    d_in = X.shape[1]
    dt = _dtype_code(X)
    if G_bp is None:
        G_bp = torch.empty(V, d_in, dtype=torch.float32, device=Z.device)
    ws = workspace(lib().dust_head_bp_grad_workspace(T, d_in, V, dt), Z.device)
    _check(lib().dust_head_bp_grad(_dev(Z, "Z", torch.float32), _dev(targets, "targets", torch.int32), _dev(X, "X"),
                                   dt, T, d_in, V, _dev(G_bp, "G_bp", torch.float32), ws.data_ptr(), ws.numel(),
                                   _stream()))
    return G_bp


def cosine(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """Device tensor of 4 doubles: (sum ab, sum aa, sum bb, cosine)."""
    if a.numel() != b.numel():
        raise ValueError("a and b must have the same number of elements")
    out = torch.empty(4, dtype=torch.float64, device=a.device)
    ws = workspace(lib().dust_cosine_workspace(), a.device)
    _check(lib().dust_cosine(_dev(a, "a", torch.float32), _dev(b, "b", torch.float32), a.numel(), out.data_ptr(),
                             ws.data_ptr(), ws.numel(), _stream()))
    return out


# ------------------------------------------------------------------ harness
def noise_fill(noise: Noise, t0: int, n_tok: int, j0: int, n_ch: int, stream_id: int = 0, device="cuda"):
    out = torch.empty(noise.draw_count, n_tok, n_ch, dtype=torch.float32, device=device)
    _check(lib().dust_noise_fill(noise.c(), stream_id, t0, n_tok, j0, n_ch, out.data_ptr(), _stream()))
    return out


def noise_sum(noise: Noise, T: int, d: int, out: torch.Tensor | None = None, device="cuda"):
    """dust_noise_sum, the generator's ceiling: out[t][j] = the sum over the
    noise's draw range of a(draw, token_begin + t, j), [T][d] fp32."""
    if out is None:
        out = torch.empty(T, d, dtype=torch.float32, device=device)
    elif tuple(out.shape) != (T, d):
        raise ValueError("out must be [T][d]")
    _check(lib().dust_noise_sum(noise.c(), T, d, _dev(out, "out", torch.float32), _stream()))
    return out


def box_muller_words(a: torch.Tensor, b: torch.Tensor):
    """Box-Muller step of the noise generator on given word pairs (uint32 held in int32 tensors)."""
    n = a.numel()
    ne = torch.empty(n, dtype=torch.float32, device=a.device)
    no = torch.empty(n, dtype=torch.float32, device=a.device)
    _check(lib().dust_box_muller_words(_dev(a, "a", torch.int32), _dev(b, "b", torch.int32), n, ne.data_ptr(),
                                       no.data_ptr(), _stream()))
    return ne, no


def synth_costs(u: torch.Tensor, noise: Noise, eps_scale: float = 0.01, out: torch.Tensor | None = None):
    T, d_out = u.shape
    c = torch.empty(noise.draw_count, T, dtype=torch.float32, device=u.device) if out is None else out
    _check(lib().dust_synth_costs(_dev(u, "u", torch.float32), T, d_out, noise.c(), float(eps_scale),
                                  _dev(c, "c", torch.float32), _stream()))
    return c


def toy_suffix_losses(Y, seq_offsets, Wq, Wk, Wv, Wo, Wout, targets, noise: Noise):
    """Returns (loss [draw_count + 1][T] with row 0 clean, c [draw_count][T])."""
    T, d = Y.shape
    dh, V = Wq.shape[0], Wout.shape[0]
    dev = Y.device
    loss = torch.empty(noise.draw_count + 1, T, dtype=torch.float32, device=dev)
    c = torch.empty(noise.draw_count, T, dtype=torch.float32, device=dev)
    ws = workspace(lib().dust_toy_suffix_workspace(noise.draw_count, T, d, dh, V), dev)
    f32 = torch.float32
    _check(lib().dust_toy_suffix_losses(_dev(Y, "Y", f32), T, d, _dev(seq_offsets, "seq_offsets", torch.int32),
                                        seq_offsets.numel() - 1, _dev(Wq, "Wq", f32), _dev(Wk, "Wk", f32),
                                        _dev(Wv, "Wv", f32), _dev(Wo, "Wo", f32), dh, _dev(Wout, "Wout", f32), V,
                                        _dev(targets, "targets", torch.int32), noise.c(), loss.data_ptr(),
                                        c.data_ptr(), ws.data_ptr(), ws.numel(), _stream()))
    return loss, c


def attention_internal_costs(Y, seq_offsets, Wq, Wk, Wv, Wo, which: int, G, noise: Noise, Wg=None, E=None):
    """Costs of the draws of `which` (0 q, 1 k, 2 v, 3 the gate's pre-activation,
    4 the value embedding) scored through the attention output against its
    estimated error G; the values are Y Wv^T + s(Y Wg^T) E: c [draw_count][T]."""
    T, d = Y.shape
    dh = Wq.shape[0]
    c = torch.empty(noise.draw_count, T, dtype=torch.float32, device=Y.device)
    ws = workspace(lib().dust_attention_internal_costs_workspace(noise.draw_count, T, d, dh), Y.device)
    f32 = torch.float32
    _check(lib().dust_attention_internal_costs(_dev(Y, "Y", f32), T, d, _dev(seq_offsets, "seq_offsets", torch.int32),
                                               seq_offsets.numel() - 1, _dev(Wq, "Wq", f32), _dev(Wk, "Wk", f32),
                                               _dev(Wv, "Wv", f32), _dev(Wo, "Wo", f32), _opt(Wg, "Wg", f32),
                                               _opt(E, "E", f32), dh, int(which), _dev(G, "G", f32), noise.c(),
                                               c.data_ptr(), ws.data_ptr(), ws.numel(), _stream()))
    return c
