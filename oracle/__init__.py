"""AB-Attention CPU oracle -- TEST INFRASTRUCTURE ONLY.

A plain double-precision restatement of the AB-Attention hot path (selector,
planner, gathered sparse forward, dense attention), written in C
(`abattn_oracle.c`) and loaded here with ctypes.  Only the tests, the
package's smoke check and the benchmark's CPU-baseline leg may import it; the
product path never does.  It shares no code with the CUDA library.

Parity pins for every function live in tests/test_oracle_*.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "abattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
u64p = np.ctypeslib.ndpointer(dtype=np.uint64, flags="C_CONTIGUOUS")
I64 = ctypes.c_int64
VP = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, -O2, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oc_meanpool.argtypes = [f64p, I64, I64, I64, f64p]
        L.oc_kmeans.argtypes = [f64p, I64, I64, ctypes.c_int, ctypes.c_int, f64p, f64p, i32p]
        L.oc_scores.argtypes = [f64p, f64p, ctypes.c_int, f64p, I64, I64, ctypes.c_double, f64p]
        L.oc_waterfill.argtypes = [f64p, I64, ctypes.c_double, f64p, ctypes.POINTER(ctypes.c_double)]
        L.oc_waterfill.restype = ctypes.c_int
        L.oc_philox4x64_10.argtypes = [u64p, u64p, u64p]
        L.oc_uniform.argtypes = [ctypes.c_uint64, I64, I64, I64, I64]
        L.oc_uniform.restype = ctypes.c_float
        L.oc_sample.argtypes = [f32p, I64, ctypes.c_uint64, I64, I64, I64, i32p, f32p, I64]
        L.oc_sample.restype = I64
        L.oc_topk.argtypes = [f64p, I64, I64, i32p]
        L.oc_topk.restype = I64
        L.oc_sparse_block.argtypes = [f64p, I64, f64p, f64p, I64, I64, I64, i32p, f32p, I64,
                                      ctypes.c_double, f64p, f64p]
        L.oc_dense.argtypes = [f64p, I64, f64p, f64p, I64, I64, ctypes.c_double, f64p, f64p]
        L.oc_selector_all.argtypes = [f64p, f64p, I64, I64, I64, I64, I64, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_double, f64p, f64p, f64p, i32p, f64p]
        L.oc_plan_all.argtypes = [f64p, I64, I64, I64, I64, ctypes.c_double, ctypes.c_int,
                                  ctypes.c_uint64, I64, VP, i64p, i32p, f32p]
        L.oc_forward_rows.argtypes = [f64p, f64p, f64p, I64, I64, I64, I64, I64, VP, I64,
                                      i64p, i32p, f32p, I64, ctypes.c_double, f64p, f64p]
        L.oc_num_threads.restype = ctypes.c_int
        L.oc_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor / array (bf16, fp32, ...) to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu")
            if x.dtype == torch.bfloat16:  # exact: a bf16 is the top half of an fp32
                bits = x.contiguous().view(torch.int16).numpy().astype(np.uint32) << 16
                return np.ascontiguousarray(bits.view(np.float32).astype(np.float64))
            return np.ascontiguousarray(x.to(torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def num_threads() -> int:
    return lib().oc_num_threads()


def set_num_threads(n: int) -> None:
    lib().oc_set_num_threads(int(n))


# ---------------------------------------------------------------- per head

def meanpool(K, kb: int) -> np.ndarray:
    """K [N, d] -> Kbar [ceil(N/kb), d]."""
    K = f64(K)
    N, d = K.shape
    out = np.empty(((N + kb - 1) // kb, d))
    lib().oc_meanpool(K, N, d, kb, out)
    return out


def kmeans(Qb, nc: int = 8, iters: int = 10):
    """Qb [M, d] -> (C [nc, d], w [nc], labels [M]); with no iterations no
    query is assigned and every label is -1."""
    Qb = f64(Qb)
    M, d = Qb.shape
    C = np.empty((nc, d))
    w = np.empty(nc)
    lab = np.full(M, -1, dtype=np.int32)
    lib().oc_kmeans(Qb, M, d, nc, iters, C, w, lab)
    return C, w, lab


def scores(C, w, Kbar, scale: float) -> np.ndarray:
    C, w, Kbar = f64(C), f64(w), f64(Kbar)
    nc, d = C.shape
    s = np.empty(Kbar.shape[0])
    lib().oc_scores(C, w, nc, Kbar, Kbar.shape[0], d, scale, s)
    return s


def waterfill(s, Bblk: float):
    """-> (pi float64, lambda, rounds)."""
    s = f64(s)
    pi = np.empty_like(s)
    lam = ctypes.c_double()
    rounds = lib().oc_waterfill(s, s.size, float(Bblk), pi, ctypes.byref(lam))
    return pi, lam.value, rounds


def philox4x64_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint64))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint64))
    out = np.empty(4, dtype=np.uint64)
    lib().oc_philox4x64_10(c, k, out)
    return out


def uniform(seed: int, b: int, h: int, qb: int, j: int) -> float:
    return lib().oc_uniform(seed, b, h, qb, j)


def sample(pi_f32, seed: int, b: int, h: int, qb: int, cap: int | None = None):
    """-> (idx int32, pi_sel float32, true count)."""
    pi = np.ascontiguousarray(np.asarray(pi_f32, dtype=np.float32))
    cap = pi.size if cap is None else cap
    idx = np.zeros(max(cap, 1), dtype=np.int32)
    ps = np.zeros(max(cap, 1), dtype=np.float32)
    n = lib().oc_sample(pi, pi.size, seed, b, h, qb, idx, ps, cap)
    m = min(n, cap)
    return idx[:m].copy(), ps[:m].copy(), n


def topk(s, k: int) -> np.ndarray:
    s = f64(s)
    idx = np.empty(max(s.size, 1), dtype=np.int32)
    n = lib().oc_topk(s, s.size, int(k), idx)
    return idx[:n].copy()


def sparse_block(Qb, K, V, kb: int, idx, pi_sel, scale: float):
    """One query block against the selected KV blocks -> (O [M, d], lse [M])."""
    Qb, K, V = f64(Qb), f64(K), f64(V)
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    ps = np.ascontiguousarray(np.asarray(pi_sel, dtype=np.float32))
    M, d = Qb.shape
    O = np.empty((M, d))
    lse = np.empty(M)
    lib().oc_sparse_block(Qb, M, K, V, K.shape[0], d, kb, idx if idx.size else np.zeros(1, np.int32),
                          ps if ps.size else np.zeros(1, np.float32), idx.size, scale, O, lse)
    return O, lse


def dense(Q, K, V, scale: float):
    """One head: Q [Nq, d], K/V [N, d] -> (O, lse)."""
    Q, K, V = f64(Q), f64(K), f64(V)
    O = np.empty_like(Q)
    lse = np.empty(Q.shape[0])
    lib().oc_dense(Q, Q.shape[0], K, V, K.shape[0], Q.shape[1], scale, O, lse)
    return O, lse


# ---------------------------------------------------------------- batched

def selector_all(Q, K, qblk: int, kb: int, nc: int, iters: int, scale: float):
    """Q, K [B, H, N, d] -> dict(Kbar, C, w, labels, S) with rows (b, h, qb)."""
    Q, K = f64(Q), f64(K)
    B, H, N, d = Q.shape
    nqb, nkvb = -(-N // qblk), -(-N // kb)
    rows = B * H * nqb
    Kbar = np.empty((B, H, nkvb, d))
    C = np.empty((B, H, nqb, nc, d))
    w = np.empty((B, H, nqb, nc))
    lab = np.full((B, H, nqb, qblk), -1, dtype=np.int32)
    S = np.empty((B, H, nqb, nkvb))
    lib().oc_selector_all(Q, K, B * H, N, d, qblk, kb, nc, iters, scale, Kbar, C, w, lab, S)
    return dict(Kbar=Kbar, C=C, w=w, labels=lab, S=S, rows=rows)


def plan_capacity(nkvb: int, budget: float) -> int:
    """Per-row capacity of a plan: min(nKVB, ceil(Bblk + 8 sqrt(Bblk) + 32))."""
    import math
    Bblk = budget * nkvb
    return int(min(nkvb, math.ceil(Bblk + 8.0 * math.sqrt(Bblk) + 32.0)))


def plan_all(S, budget: float, mode: int, seed: int, cap: int | None = None, want_pi=False):
    """S [B, H, nqb, nkvb] -> dict(counts, idx, pi_sel[, pi])."""
    S = f64(S)
    B, H, nqb, nkvb = S.shape
    cap = plan_capacity(nkvb, budget) if cap is None else cap
    rows = B * H * nqb
    counts = np.empty(rows, dtype=np.int64)
    idx = np.zeros((rows, cap), dtype=np.int32)
    ps = np.zeros((rows, cap), dtype=np.float32)
    pi = np.empty((rows, nkvb), dtype=np.float32) if want_pi else None
    lib().oc_plan_all(S, B, H, nqb, nkvb, budget * nkvb, mode, seed, cap,
                      pi.ctypes.data if want_pi else None, counts, idx, ps)
    out = dict(counts=counts.reshape(B, H, nqb), idx=idx.reshape(B, H, nqb, cap),
               pi_sel=ps.reshape(B, H, nqb, cap), cap=cap)
    if want_pi:
        out["pi"] = pi.reshape(B, H, nqb, nkvb)
    return out


def forward_rows(Q, K, V, qblk: int, kb: int, counts, idx, pi_sel, scale: float, rows=None,
                 O=None, lse=None):
    """Sparse forward for `rows` (flat ids b*H*nqb + h*nqb + qb; None = all).

    counts/idx/pi_sel hold one plan row per listed row (all rows when rows is
    None).  Returns (O [B, H, N, d], lse [B, H, N]) with unlisted rows zero.
    """
    Q, K, V = f64(Q), f64(K), f64(V)
    B, H, N, d = Q.shape
    nqb = -(-N // qblk)
    counts = np.ascontiguousarray(np.asarray(counts, dtype=np.int64).reshape(-1))
    cap = np.asarray(idx).shape[-1]
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(-1, cap))
    pi_sel = np.ascontiguousarray(np.asarray(pi_sel, dtype=np.float32).reshape(-1, cap))
    if O is None:
        O = np.zeros((B, H, N, d))
    if lse is None:
        lse = np.zeros((B, H, N))
    if rows is None:
        n_rows, rp = B * H * nqb, None
    else:
        rarr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n_rows, rp = rarr.size, rarr.ctypes.data
    lib().oc_forward_rows(Q, K, V, B * H, N, d, qblk, kb, rp, n_rows, counts, idx, pi_sel, cap,
                          scale, O, lse)
    return O, lse


def plan_forward_row(Qh, Kh, Vh, Kbar_h, b: int, h: int, qb: int, kb: int, budget: float, seed: int,
                     nc: int = 8, iters: int = 10, scale: float | None = None, mode: int = 0):
    """The whole path for one q-block row of one head, step by step:
    k-means of the row's queries, scores against the head's mean keys,
    water-fill + Poisson sampling (or top-k), then the gathered forward.
    Qh, Kh, Vh: float64 [N, d] of the head; Kbar_h: its mean keys.
    Returns dict(O, lse, idx, pi_sel, S)."""
    Qh, Kh, Vh = f64(Qh), f64(Kh), f64(Vh)
    N, d = Qh.shape
    scale = 1.0 / (d ** 0.5) if scale is None else scale
    q0 = qb * 128
    Qb = np.ascontiguousarray(Qh[q0:q0 + 128])
    C, w, _ = kmeans(Qb, nc, iters)
    s = scores(C, w, Kbar_h, scale)
    nkvb = s.size
    if mode == 0:
        pi, _, _ = waterfill(s, budget * nkvb)
        idx, ps, _ = sample(pi.astype(np.float32), seed, b, h, qb)
    else:
        idx = topk(s, int(np.floor(budget * nkvb + 0.5)))
        ps = np.ones(idx.size, dtype=np.float32)
    O, lse = sparse_block(Qb, Kh, Vh, kb, idx, ps, scale)
    return dict(O=O, lse=lse, idx=idx, pi_sel=ps, S=s)


# ---------------------------------------------------------------- 8-bit forward inputs
# The FP8 E4M3 forward (VC-Attention pages, B200 results: 8-bit attention on
# Blackwell) quantises Q per 128-query block and K per KV block, each block
# with its own scale.  E4M3 is the OCP 8-bit float with one sign bit, four
# exponent bits (bias 7) and three mantissa bits; its largest finite value is
# 448, and there is no infinity.  A block's scale is amax / 448, so that its
# largest element maps to the largest code; a block of zeros takes scale 1.

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 byte codes -> float64, from the format definition (NaN for the two
    NaN codes 0x7F and 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    val = sign * val
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


def e4m3_encode(x) -> np.ndarray:
    """float32 values already inside [-448, 448] -> E4M3 codes, rounded to
    nearest even (torch's float8_e4m3fn conversion as the rounding step)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(x, dtype=np.float32)))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()


def quantize_e4m3_rows(X, rows_per_block: int):
    """X [..., n, d] (the bf16 values as float32) -> (codes uint8 [..., n, d],
    scales float32 [..., ceil(n / rows_per_block)]).

    Per block of rows_per_block consecutive rows (the last one may be short):
    amax = max |x| over the block; scale = fp32(amax / 448) and
    inv = fp32(448 / amax) (1 and 1 for an all-zero block); each element is
    encoded from fp32(x * inv), clamped to +-448 against the rounding of inv."""
    X = np.asarray(X, dtype=np.float32)
    *lead, n, d = X.shape
    nb = -(-n // rows_per_block)
    pad = nb * rows_per_block - n
    Xp = np.concatenate([X, np.zeros((*lead, pad, d), np.float32)], axis=-2) if pad else X
    blocks = Xp.reshape(*lead, nb, rows_per_block, d)
    amax = np.abs(blocks).max(axis=(-2, -1))
    zero = amax == 0
    safe = np.where(zero, np.float32(1), amax).astype(np.float32)
    scale = np.where(zero, np.float32(1), (safe / np.float32(E4M3_MAX)).astype(np.float32)).astype(np.float32)
    inv = np.where(zero, np.float32(1), (np.float32(E4M3_MAX) / safe).astype(np.float32)).astype(np.float32)
    y = (blocks * inv[..., None, None]).astype(np.float32)
    y = np.clip(y, -E4M3_MAX, E4M3_MAX).astype(np.float32)
    codes = e4m3_encode(y).reshape(*lead, nb * rows_per_block, d)[..., :n, :]
    return np.ascontiguousarray(codes), scale


def dequantize_e4m3_rows(codes, scales, rows_per_block: int) -> np.ndarray:
    """Inverse of quantize_e4m3_rows up to the rounding: code value x block
    scale, in float64."""
    v = e4m3_decode(codes)
    *lead, n, d = v.shape
    rep = np.repeat(np.asarray(scales, dtype=np.float64), rows_per_block, axis=-1)[..., :n]
    return v * rep[..., None]
