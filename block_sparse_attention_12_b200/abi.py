"""ctypes binding of libabattn.so (include/abattn.h).

Argument marshalling only: every step of the AB-Attention path runs in the
library's CUDA kernels.  torch is used to allocate device buffers and to
name the current stream.  If the library is missing the first call raises;
there is no other code path.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libabattn.so")

OK = 0
ERR_NULL, ERR_SHAPE, ERR_PARAM, ERR_ALIGN, ERR_WORKSPACE = -1, -2, -3, -4, -5
ERR_PLAN_OVERFLOW, ERR_TIMEOUT, ERR_BOUNDS, ERR_CUDA, ERR_DEVICE = -6, -7, -8, -9, -10
MODE_SIP, MODE_TOPK = 0, 1

EXPORTED = [
    "abattn_version", "abattn_strerror", "abattn_check", "abattn_plan_capacity",
    "abattn_plan_workspace_size", "abattn_score_workspace_size", "abattn_meanpool",
    "abattn_kmeans", "abattn_score", "abattn_plan_from_scores", "abattn_plan_from_pi",
    "abattn_plan", "abattn_forward", "abattn_dense_forward", "abattn_plan_noalloc",
    "abattn_quantize_e4m3", "abattn_forward_e4m3",
]


def _header_define(name: str) -> int:
    """Integer value of a `#define NAME (a << b)` or `#define NAME n` in
    include/abattn.h, so that the binding and the library share one value."""
    import re
    path = os.path.join(os.path.dirname(_HERE), "include", "abattn.h")
    with open(path) as f:
        m = re.search(r"#define\s+" + name + r"\s+\((\d+)u?\s*<<\s*(\d+)\)|#define\s+" + name + r"\s+(\d+)",
                      f.read())
    if m is None:
        raise RuntimeError(f"{name} not found in {path}")
    return int(m.group(1)) << int(m.group(2)) if m.group(1) else int(m.group(3))


NOALLOC_SCRATCH_BYTES = _header_define("ABATTN_NOALLOC_SCRATCH_BYTES")


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("N", ctypes.c_int64),
                ("d", ctypes.c_int64)]


class Params(ctypes.Structure):
    _fields_ = [("q_block", ctypes.c_int32), ("kv_block", ctypes.c_int32),
                ("n_clusters", ctypes.c_int32), ("kmeans_iters", ctypes.c_int32),
                ("budget", ctypes.c_float), ("mode", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("scale", ctypes.c_float), ("head_offset", ctypes.c_int32)]


class AbattnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {strerror(code)} ({code})")
        self.code = code


_lib = None
VP = ctypes.c_void_p
P_D = ctypes.POINTER(Dims)
P_P = ctypes.POINTER(Params)


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"AB-Attention CUDA library not built: {LIB_PATH} missing "
                               "(run block_sparse_attention_12_b200.build.build())")
        L = ctypes.CDLL(LIB_PATH)
        L.abattn_version.restype = ctypes.c_char_p
        L.abattn_strerror.restype = ctypes.c_char_p
        L.abattn_strerror.argtypes = [ctypes.c_int]
        L.abattn_check.argtypes = [VP]
        L.abattn_plan_capacity.argtypes = [P_D, P_P, ctypes.POINTER(ctypes.c_int64)]
        L.abattn_plan_workspace_size.argtypes = [P_D, P_P, ctypes.POINTER(ctypes.c_size_t)]
        L.abattn_score_workspace_size.argtypes = [P_D, P_P, ctypes.POINTER(ctypes.c_size_t)]
        L.abattn_meanpool.argtypes = [VP, P_D, ctypes.c_int32, VP, VP]
        L.abattn_kmeans.argtypes = [VP, P_D, P_P, VP, VP, VP, VP]
        L.abattn_score.argtypes = [VP, VP, VP, P_D, P_P, VP, VP, ctypes.c_size_t, VP]
        L.abattn_plan_from_scores.argtypes = [VP, P_D, P_P, VP, VP, VP, ctypes.c_int64, VP, VP]
        L.abattn_plan_from_pi.argtypes = [VP, P_D, P_P, VP, VP, VP, ctypes.c_int64, VP]
        L.abattn_plan.argtypes = [VP, VP, P_D, P_P, VP, VP, VP, ctypes.c_int64, VP, ctypes.c_size_t, VP]
        L.abattn_forward.argtypes = [VP, VP, VP, P_D, P_P, VP, VP, VP, ctypes.c_int64, VP, VP, VP]
        L.abattn_dense_forward.argtypes = [VP, VP, VP, P_D, ctypes.c_float, VP, VP, VP]
        L.abattn_plan_noalloc.argtypes = [VP, VP, P_D, P_P, VP, VP, VP, ctypes.c_int64, VP]
        L.abattn_quantize_e4m3.argtypes = [VP, P_D, ctypes.c_int, VP, VP, VP]
        L.abattn_forward_e4m3.argtypes = [VP, VP, VP, VP, VP, P_D, P_P, VP, VP, VP, ctypes.c_int64, VP, VP, VP]
        for name in EXPORTED:
            if name not in ("abattn_version", "abattn_strerror"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().abattn_strerror(int(code)).decode()


def version() -> str:
    return lib().abattn_version().decode()


def _ok(code: int, where: str) -> None:
    if code != OK:
        raise AbattnError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclasses.dataclass
class Config:
    """The method's knobs (kv_block 4, 8 clusters, 10 Lloyd iterations)."""

    kv_block: int = 4
    budget: float = 0.08
    n_clusters: int = 8
    kmeans_iters: int = 10
    mode: int = MODE_SIP
    seed: int = 0
    scale: float = 0.0
    q_block: int = 128
    head_offset: int = 0  # global index of the first head when the tensors hold a slice of a layer's heads

    def params(self) -> Params:
        return Params(self.q_block, self.kv_block, self.n_clusters, self.kmeans_iters,
                      float(self.budget), self.mode, self.seed, float(self.scale), self.head_offset)


def dims_of(Q: torch.Tensor) -> Dims:
    B, H, N, d = Q.shape
    return Dims(B, H, N, d)


@dataclasses.dataclass
class Plan:
    counts: torch.Tensor   # int32 [B, H, nQB]
    idx: torch.Tensor      # int32 [B, H, nQB, cap]
    pi_sel: torch.Tensor   # fp32  [B, H, nQB, cap]
    cap: int
    kv_block: int


def _check_qkv(*ts):
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4 or not t.is_cuda:
            raise ValueError("Q, K, V must be contiguous CUDA bf16 tensors [B, H, N, d]")


def capacity(shape, cfg: Config) -> int:
    B, H, N, d = shape
    cap = ctypes.c_int64()
    _ok(lib().abattn_plan_capacity(ctypes.byref(Dims(B, H, N, d)), ctypes.byref(cfg.params()),
                                   ctypes.byref(cap)), "abattn_plan_capacity")
    return cap.value


def plan_workspace_bytes(shape, cfg: Config) -> int:
    n = ctypes.c_size_t()
    _ok(lib().abattn_plan_workspace_size(ctypes.byref(Dims(*shape)), ctypes.byref(cfg.params()),
                                         ctypes.byref(n)), "abattn_plan_workspace_size")
    return n.value


def score_workspace_bytes(shape, cfg: Config) -> int:
    n = ctypes.c_size_t()
    _ok(lib().abattn_score_workspace_size(ctypes.byref(Dims(*shape)), ctypes.byref(cfg.params()),
                                          ctypes.byref(n)), "abattn_score_workspace_size")
    return n.value


def empty_plan(shape, cfg: Config, device="cuda") -> Plan:
    B, H, N, d = shape
    nqb = -(-N // 128)
    cap = capacity(shape, cfg)
    return Plan(torch.zeros(B, H, nqb, dtype=torch.int32, device=device),
                torch.zeros(B, H, nqb, cap, dtype=torch.int32, device=device),
                torch.zeros(B, H, nqb, cap, dtype=torch.float32, device=device), cap, cfg.kv_block)


def meanpool(K: torch.Tensor, kv_block: int, out=None, stream=None) -> torch.Tensor:
    _check_qkv(K)
    B, H, N, d = K.shape
    if out is None:
        out = torch.empty(B, H, -(-N // kv_block), d, dtype=torch.float32, device=K.device)
    _ok(lib().abattn_meanpool(_ptr(K), ctypes.byref(dims_of(K)), kv_block, _ptr(out), _stream(stream)),
        "abattn_meanpool")
    return out


def kmeans(Q: torch.Tensor, cfg: Config, stream=None):
    _check_qkv(Q)
    B, H, N, d = Q.shape
    nqb = -(-N // 128)
    C = torch.empty(B, H, nqb, cfg.n_clusters, d, dtype=torch.float32, device=Q.device)
    w = torch.empty(B, H, nqb, cfg.n_clusters, dtype=torch.float32, device=Q.device)
    lab = torch.empty(B, H, nqb, 128, dtype=torch.int32, device=Q.device)
    _ok(lib().abattn_kmeans(_ptr(Q), ctypes.byref(dims_of(Q)), ctypes.byref(cfg.params()), _ptr(C), _ptr(w),
                            _ptr(lab), _stream(stream)), "abattn_kmeans")
    return C, w, lab


def score(C, w, Kbar, shape, cfg: Config, stream=None):
    B, H, N, d = shape
    nqb, nkvb = -(-N // 128), -(-N // cfg.kv_block)
    C, w, Kbar = C.contiguous().float(), w.contiguous().float(), Kbar.contiguous().float()
    S = torch.empty(B, H, nqb, nkvb, dtype=torch.float32, device=C.device)
    ws = torch.empty(score_workspace_bytes(shape, cfg), dtype=torch.uint8, device=C.device)
    _ok(lib().abattn_score(_ptr(C), _ptr(w), _ptr(Kbar), ctypes.byref(Dims(*shape)),
                           ctypes.byref(cfg.params()), _ptr(S), _ptr(ws), ws.numel(), _stream(stream)),
        "abattn_score")
    return S


def plan_from_scores(S, shape, cfg: Config, want_pi=False, plan=None, stream=None):
    S = S.contiguous().float()
    plan = empty_plan(shape, cfg, S.device) if plan is None else plan
    pi = torch.empty_like(S) if want_pi else None
    _ok(lib().abattn_plan_from_scores(_ptr(S), ctypes.byref(Dims(*shape)), ctypes.byref(cfg.params()),
                                      _ptr(plan.counts), _ptr(plan.idx), _ptr(plan.pi_sel), plan.cap,
                                      _ptr(pi), _stream(stream)), "abattn_plan_from_scores")
    return (plan, pi) if want_pi else plan


def plan_from_pi(pi, shape, cfg: Config, plan=None, stream=None):
    pi = pi.contiguous().float()
    plan = empty_plan(shape, cfg, pi.device) if plan is None else plan
    _ok(lib().abattn_plan_from_pi(_ptr(pi), ctypes.byref(Dims(*shape)), ctypes.byref(cfg.params()),
                                  _ptr(plan.counts), _ptr(plan.idx), _ptr(plan.pi_sel), plan.cap,
                                  _stream(stream)), "abattn_plan_from_pi")
    return plan


class Planner:
    """Holds the plan workspace so repeated plans allocate nothing."""

    def __init__(self, shape, cfg: Config, device="cuda"):
        self.shape, self.cfg = tuple(shape), cfg
        self.ws = torch.empty(plan_workspace_bytes(self.shape, cfg), dtype=torch.uint8, device=device)
        self.plan = empty_plan(self.shape, cfg, device)

    def __call__(self, Q, K, stream=None) -> Plan:
        _check_qkv(Q, K)
        p = self.plan
        _ok(lib().abattn_plan(_ptr(Q), _ptr(K), ctypes.byref(Dims(*self.shape)), ctypes.byref(self.cfg.params()),
                              _ptr(p.counts), _ptr(p.idx), _ptr(p.pi_sel), p.cap, _ptr(self.ws),
                              self.ws.numel(), _stream(stream)), "abattn_plan")
        return p


def plan(Q, K, cfg: Config, stream=None) -> Plan:
    return Planner(Q.shape, cfg, Q.device)(Q, K, stream)


def plan_noalloc(Q, K, cfg: Config, plan: Plan | None = None, stream=None) -> Plan:
    """abattn_plan_noalloc: the same plan as `plan`, with the library's own
    fixed scratch array instead of a caller workspace (small layers only).
    The output buffers are still the caller's (allocated here when `plan` is
    None)."""
    _check_qkv(Q, K)
    p = empty_plan(Q.shape, cfg, Q.device) if plan is None else plan
    _ok(lib().abattn_plan_noalloc(_ptr(Q), _ptr(K), ctypes.byref(dims_of(Q)), ctypes.byref(cfg.params()),
                                  _ptr(p.counts), _ptr(p.idx), _ptr(p.pi_sel), p.cap, _stream(stream)),
        "abattn_plan_noalloc")
    return p


def forward(Q, K, V, plan: Plan, cfg: Config | None = None, O=None, lse=None, want_lse=True, stream=None):
    _check_qkv(Q, K, V)
    cfg = cfg or Config(kv_block=plan.kv_block)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=Q.device)
    _ok(lib().abattn_forward(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(dims_of(Q)), ctypes.byref(cfg.params()),
                             _ptr(plan.counts), _ptr(plan.idx), _ptr(plan.pi_sel), plan.cap, _ptr(O), _ptr(lse),
                             _stream(stream)), "abattn_forward")
    return O, lse


def quantize_e4m3(X, rows_per_block: int, codes=None, scales=None, stream=None):
    """bf16 [B, H, N, 128] -> (E4M3 codes uint8 [B, H, N, 128], scales fp32
    [B, H, ceil(N / rows_per_block)]), one scale per block of rows (128 rows for
    Q, the plan's kv_block for K)."""
    _check_qkv(X)
    B, H, N, d = X.shape
    if codes is None:
        codes = torch.empty(B, H, N, d, dtype=torch.uint8, device=X.device)
    if scales is None:
        scales = torch.empty(B, H, -(-N // rows_per_block), dtype=torch.float32, device=X.device)
    _ok(lib().abattn_quantize_e4m3(_ptr(X), ctypes.byref(dims_of(X)), int(rows_per_block), _ptr(codes),
                                   _ptr(scales), _stream(stream)), "abattn_quantize_e4m3")
    return codes, scales


def forward_e4m3(Q8, q_scales, K8, k_scales, V, plan: Plan, cfg: Config | None = None, O=None, lse=None,
                 want_lse=True, stream=None):
    """The gathered sparse forward with QK^T in E4M3 (Q8, K8 and their scales
    from quantize_e4m3: 128 rows per block for Q, the plan's kv_block for K);
    V bf16 [B, H, N, 128]."""
    _check_qkv(V)
    for t in (Q8, K8):
        if t.dtype != torch.uint8 or t.shape != V.shape or not t.is_contiguous():
            raise ValueError("E4M3 codes must be contiguous uint8 tensors shaped like V")
    cfg = cfg or Config(kv_block=plan.kv_block)
    if O is None:
        O = torch.empty_like(V)
    if lse is None and want_lse:
        lse = torch.empty(V.shape[:3], dtype=torch.float32, device=V.device)
    _ok(lib().abattn_forward_e4m3(_ptr(Q8), _ptr(q_scales), _ptr(K8), _ptr(k_scales), _ptr(V),
                                  ctypes.byref(dims_of(V)), ctypes.byref(cfg.params()), _ptr(plan.counts),
                                  _ptr(plan.idx), _ptr(plan.pi_sel), plan.cap, _ptr(O), _ptr(lse),
                                  _stream(stream)), "abattn_forward_e4m3")
    return O, lse


def dense_forward(Q, K, V, scale: float = 0.0, O=None, lse=None, want_lse=True, stream=None):
    _check_qkv(Q, K, V)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=Q.device)
    _ok(lib().abattn_dense_forward(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(dims_of(Q)), float(scale), _ptr(O),
                                   _ptr(lse), _stream(stream)), "abattn_dense_forward")
    return O, lse


def check(stream=None) -> None:
    """Synchronises and raises if a kernel reported an error."""
    _ok(lib().abattn_check(_stream(stream)), "abattn_check")


def full_plan(shape, kv_block: int, device="cuda") -> Plan:
    """Every KV block with weight 1 (the full-budget plan)."""
    B, H, N, d = shape
    nqb, nkvb = -(-N // 128), -(-N // kv_block)
    idx = torch.arange(nkvb, dtype=torch.int32, device=device).expand(B, H, nqb, nkvb).contiguous()
    return Plan(torch.full((B, H, nqb), nkvb, dtype=torch.int32, device=device), idx,
                torch.ones(B, H, nqb, nkvb, dtype=torch.float32, device=device), nkvb, kv_block)


def executed_flops(plan: Plan, shape) -> float:
    """Tensor-core FLOPs the sparse forward issues: every 128-key tile is a
    full 128x128 QK^T and PV, padded slots included."""
    B, H, N, d = shape
    keys = plan.counts.to(torch.int64) * plan.kv_block
    tiles = (keys + 127) // 128
    return float(4.0 * 128 * 128 * d * tiles.sum().item())


def useful_flops(plan: Plan, shape) -> float:
    """FLOPs of the selected keys only: 4 d M_qb (kb n_sel), M_qb the q-block's
    true query count."""
    B, H, N, d = shape
    nqb = -(-N // 128)
    M = torch.full((nqb,), 128, dtype=torch.int64)
    M[-1] = N - 128 * (nqb - 1)
    keys = plan.counts.to("cpu", torch.int64) * plan.kv_block
    return float(4.0 * d * (keys * M).sum().item())
