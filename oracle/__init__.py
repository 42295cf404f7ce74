"""CPU oracle for the Dust estimator hot path (numpy front end over liboracle.so).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package.  It shares no code with the CUDA
library: the noise specification is implemented here (in C) independently.

Every function takes and returns numpy arrays; floating-point results are
float64 except the noise itself, which is binary32 by specification.
"""
from __future__ import annotations

import ctypes as C
import numpy as np

from .build import build

_lib = None

_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")


def _nullable(kind):
    """ndpointer that also accepts None (NULL)."""
    class _P(kind):  # type: ignore[misc, valid-type]
        @classmethod
        def from_param(cls, obj):
            if obj is None:
                return None
            return super().from_param(obj)
    return _P


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def load(path: str) -> C.CDLL:
    """Load an oracle library built from these sources (the tests also load
    deliberately broken builds, to show that the pins catch them)."""
    L = C.CDLL(path)
    u32, i32, dbl, flt = C.c_uint32, C.c_int, C.c_double, C.c_float
    L.orc_philox4x32_10.argtypes = [_u32p, _u32p, _u32p]
    L.orc_ln.argtypes = [flt]
    L.orc_ln.restype = flt
    L.orc_sincos_quarter.argtypes = [flt, C.POINTER(flt), C.POINTER(flt)]
    L.orc_box_muller.argtypes = [u32, u32, C.POINTER(flt), C.POINTER(flt)]
    L.orc_philox_batch.argtypes = [_u32p, _u32p, i32, _u32p]
    L.orc_ln_batch.argtypes = [_f32p, i32, _f32p]
    L.orc_sincos_batch.argtypes = [_f32p, i32, _f32p, _f32p]
    L.orc_box_muller_batch.argtypes = [_u32p, _u32p, i32, _f32p, _f32p]
    L.orc_gauss.argtypes = [u32] * 6
    L.orc_gauss.restype = flt
    L.orc_noise_block.argtypes = [u32, u32, u32, u32, i32, _i32p, i32, u32, i32, _f32p]
    L.orc_reward_scan.argtypes = [_f32p, _f64p, i32, i32, _i32p, i32, dbl]
    L.orc_reward_scan.restype = i32
    L.orc_reward_scan_brute.argtypes = [_f32p, _f64p, i32, i32, _i32p, i32, dbl]
    L.orc_reward_scan_brute.restype = i32
    L.orc_layer_estimate.argtypes = [_f32p, i32, i32, i32, i32, _i32p, i32, dbl,
                                     u32, u32, u32, u32, i32, dbl, _i32p, i32,
                                     _nullable(_i32p), i32, _f64p]
    L.orc_layer_estimate.restype = i32
    L.orc_weight_grad.argtypes = [_f32p, _f32p, i32, i32, i32, _i32p, i32, _f64p]
    L.orc_weight_grad.restype = i32
    L.orc_logits.argtypes = [_f32p, _f32p, i32, i32, i32, _i32p, i32, _f64p]
    L.orc_logits.restype = i32
    L.orc_head_clean.argtypes = [_f32p, _i32p, i32, i32, _f64p, _f64p]
    L.orc_head_clean.restype = i32
    L.orc_head_step.argtypes = [_f32p, _i32p, _i32p, i32, i32, i32, u32, u32, u32, i32,
                                i32, dbl, _nullable(_f64p), _f64p]
    L.orc_head_step.restype = i32
    L.orc_head_bp_grad.argtypes = [_f32p, _i32p, _f32p, i32, i32, i32, _i32p, i32, _f64p]
    L.orc_head_bp_grad.restype = i32
    L.orc_cosine.argtypes = [_f32p, _f32p, C.c_longlong]
    L.orc_cosine.restype = dbl
    L.orc_synth_costs.argtypes = [_f32p, i32, i32, u32, u32, dbl, dbl, _i32p, _i32p, i32, _f64p]
    L.orc_synth_costs.restype = i32
    L.orc_toy_suffix_losses.argtypes = [_f32p, _f32p, i32, i32, i32, _i32p, i32,
                                        _f32p, _f32p, _f32p, _f32p, i32, _f32p, i32,
                                        _i32p, u32, u32, dbl, i32, _i32p, i32, _f64p]
    L.orc_toy_suffix_losses.restype = i32
    L.orc_attention_internal_costs.argtypes = [_f32p, i32, i32, _i32p, i32, _f32p, _f32p, _f32p, _f32p,
                                               _nullable(_f32p), _nullable(_f32p), i32, i32,
                                               _f32p, u32, u32, dbl, _i32p, i32, _f64p]
    L.orc_attention_internal_costs.restype = i32
    return L


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


# ---------------------------------------------------------------- noise

def philox4x32_10(ctr, key) -> np.ndarray:
    out = np.zeros(4, np.uint32)
    lib().orc_philox4x32_10(np.asarray(ctr, np.uint32), np.asarray(key, np.uint32), out)
    return out


def ln(u: float) -> np.float32:
    return np.float32(lib().orc_ln(C.c_float(u)))


def sincos_quarter(phi: float):
    s, c = C.c_float(), C.c_float()
    lib().orc_sincos_quarter(C.c_float(phi), C.byref(s), C.byref(c))
    return np.float32(s.value), np.float32(c.value)


def box_muller(a: int, b: int):
    e, o = C.c_float(), C.c_float()
    lib().orc_box_muller(a, b, C.byref(e), C.byref(o))
    return np.float32(e.value), np.float32(o.value)


def philox_batch(ctr, key) -> np.ndarray:
    """ctr [n][4], key [n][2] (uint32) -> [n][4]."""
    ctr = np.ascontiguousarray(ctr, np.uint32)
    key = np.ascontiguousarray(key, np.uint32)
    out = np.zeros_like(ctr)
    lib().orc_philox_batch(ctr, key, len(ctr), out)
    return out


def ln_batch(u) -> np.ndarray:
    u = _f32(u)
    out = np.zeros_like(u)
    lib().orc_ln_batch(u, u.size, out)
    return out


def sincos_batch(phi):
    phi = _f32(phi)
    s = np.zeros_like(phi)
    c = np.zeros_like(phi)
    lib().orc_sincos_batch(phi, phi.size, s, c)
    return s, c


def box_muller_batch(a, b):
    a = np.ascontiguousarray(a, np.uint32)
    b = np.ascontiguousarray(b, np.uint32)
    ne = np.zeros(a.shape, np.float32)
    no = np.zeros(a.shape, np.float32)
    lib().orc_box_muller_batch(a, b, a.size, ne, no)
    return ne, no


def gauss(seed, layer, draw, token, channel, stream=0) -> np.float32:
    return np.float32(lib().orc_gauss(seed, layer, draw, token, channel, stream))


def noise_block(seed, layer, draw0, nd, tokens, ch0, nc, stream=0) -> np.ndarray:
    """[nd][len(tokens)][nc] binary32 noise."""
    tokens = _i32(tokens)
    out = np.zeros((nd, len(tokens), nc), np.float32)
    lib().orc_noise_block(seed, layer, stream, draw0, nd, tokens, len(tokens), ch0, nc, out)
    return out


# ---------------------------------------------------------------- a4 / a5 / a6

def reward_scan(c, seq_offsets, gamma, brute=False) -> np.ndarray:
    c = _f32(c)
    K, T = c.shape
    off = _i32(seq_offsets)
    r = np.zeros((K, T), np.float64)
    f = lib().orc_reward_scan_brute if brute else lib().orc_reward_scan
    _check(f(c, r, K, T, off, len(off) - 1, float(gamma)), "reward_scan")
    return r


def layer_estimate(c_or_r, is_r, d_out, seq_offsets, gamma, seed, layer, draw_begin,
                   K_total, sigma, toks, chans=None, token_begin=0) -> np.ndarray:
    """g[len(toks)][len(chans) or d_out] in float64; c_or_r is [K][T] float32;
    column t draws the noise of global token token_begin + t."""
    a = _f32(c_or_r)
    K, T = a.shape
    off = _i32(seq_offsets)
    toks = _i32(toks)
    chans_a = None if chans is None else _i32(chans)
    nc = d_out if chans is None else len(chans_a)
    g = np.zeros((len(toks), nc), np.float64)
    _check(lib().orc_layer_estimate(a, int(bool(is_r)), K, T, d_out, off, len(off) - 1,
                                    float(gamma), seed, layer, draw_begin, int(token_begin), K_total, float(sigma),
                                    toks, len(toks), chans_a, nc, g), "layer_estimate")
    return g


def weight_grad(g, X, rows=None) -> np.ndarray:
    g = _f32(g)
    X = _f32(X)
    T, d_out = g.shape
    d_in = X.shape[1]
    rows = _i32(np.arange(d_out) if rows is None else rows)
    G = np.zeros((len(rows), d_in), np.float64)
    _check(lib().orc_weight_grad(g, X, T, d_in, d_out, rows, len(rows), G), "weight_grad")
    return G


def synth_costs(u, seed, layer, sigma, eps_scale, draws, toks) -> np.ndarray:
    u = _f32(u)
    T, d_out = u.shape
    draws = _i32(draws)
    toks = _i32(toks)
    c = np.zeros(len(draws), np.float64)
    _check(lib().orc_synth_costs(u, T, d_out, seed, layer, float(sigma), float(eps_scale),
                                 draws, toks, len(draws), c), "synth_costs")
    return c


# ---------------------------------------------------------------- head

def logits(X, W, toks=None) -> np.ndarray:
    X = _f32(X)
    W = _f32(W)
    T, d_in = X.shape
    V = W.shape[0]
    toks = _i32(np.arange(T) if toks is None else toks)
    Z = np.zeros((len(toks), V), np.float64)
    _check(lib().orc_logits(X, W, T, d_in, V, toks, len(toks), Z), "logits")
    return Z


def head_clean(Zrows, y):
    Zrows = _f32(Zrows)
    n, V = Zrows.shape
    lse = np.zeros(n, np.float64)
    ell = np.zeros(n, np.float64)
    _check(lib().orc_head_clean(Zrows, _i32(y), n, V, lse, ell), "head_clean")
    return lse, ell


def head_step(Zrows, y, toks, Vc, seed, layer, draw_begin, nd, K_total, sigma, want_c=True):
    """Returns (c [V/Vc][nd][n] or None, g [n][V]) in float64."""
    Zrows = _f32(Zrows)
    n, V = Zrows.shape
    c = np.zeros((V // Vc, nd, n), np.float64) if want_c else None
    g = np.zeros((n, V), np.float64)
    _check(lib().orc_head_step(Zrows, _i32(y), _i32(toks), n, V, Vc, seed, layer, draw_begin,
                               nd, K_total, float(sigma), c, g), "head_step")
    return c, g


def head_bp_grad(Z, y, X, rows=None) -> np.ndarray:
    """Backprop gradient of sum_t CE(z_t, y_t) w.r.t. W (rows of [V][d_in]), float64."""
    Z = _f32(Z)
    X = _f32(X)
    T, V = Z.shape
    d_in = X.shape[1]
    rows = _i32(np.arange(V) if rows is None else rows)
    G = np.zeros((len(rows), d_in), np.float64)
    _check(lib().orc_head_bp_grad(Z, _i32(y), X, T, d_in, V, rows, len(rows), G), "head_bp_grad")
    return G


def cosine(a, b) -> float:
    a = _f32(np.ravel(a))
    b = _f32(np.ravel(b))
    return float(lib().orc_cosine(a, b, a.size))


# ---------------------------------------------------------------- toy suffix

def toy_suffix_losses(X, W, seq_offsets, Wq, Wk, Wv, Wo, Wout, targets, seed, layer,
                      sigma, draws, with_noise=True) -> np.ndarray:
    X, W, Wq, Wk, Wv, Wo, Wout = (_f32(a) for a in (X, W, Wq, Wk, Wv, Wo, Wout))
    T, d_in = X.shape
    d = W.shape[0]
    dh = Wq.shape[0]
    V = Wout.shape[0]
    off = _i32(seq_offsets)
    draws = _i32(draws)
    loss = np.zeros((len(draws), T), np.float64)
    _check(lib().orc_toy_suffix_losses(X, W, T, d_in, d, off, len(off) - 1, Wq, Wk, Wv, Wo, dh,
                                       Wout, V, _i32(targets), seed, layer, float(sigma),
                                       int(bool(with_noise)), draws, len(draws), loss),
           "toy_suffix_losses")
    return loss


# ---------------------------------------------------------------- attention-internal scoring

def attention_internal_costs(Y, seq_offsets, Wq, Wk, Wv, Wo, which, G, seed, layer, sigma, draws,
                             Wg=None, E=None) -> np.ndarray:
    """c[n][t] = -<z~_t - z_t, G_t> for perturbations of `which` (0 q, 1 k, 2 v, 3 the
    gate's pre-activation, 4 the value embedding); values v = Y Wv^T + s(Y Wg^T) E."""
    Y, Wq, Wk, Wv, Wo, G = (_f32(a) for a in (Y, Wq, Wk, Wv, Wo, G))
    Wg = None if Wg is None else _f32(Wg)
    E = None if E is None else _f32(E)
    T, d = Y.shape
    dh = Wq.shape[0]
    off = _i32(seq_offsets)
    draws = _i32(draws)
    c = np.zeros((len(draws), T), np.float64)
    _check(lib().orc_attention_internal_costs(Y, T, d, off, len(off) - 1, Wq, Wk, Wv, Wo, Wg, E, dh, int(which), G,
                                              seed, layer, float(sigma), draws, len(draws), c),
           "attention_internal_costs")
    return c
