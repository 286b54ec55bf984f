"""ctypes binding of liblora_mlp.so (include/lora_mlp.h): argument marshalling only.

Every step of the LoRA-MLP path runs in the library's CUDA kernels; torch is used
here only to allocate device memory and to name the current stream.  If the
library is missing the import fails loudly: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblora_mlp.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "lora_mlp.h")

LORA_OK = 0
ERRORS = {-1: "INVALID_ARG", -2: "ALIGNMENT", -3: "UNSUPPORTED", -4: "CUDA", -5: "TIMEOUT"}
WFMT_BF16, WFMT_4BIT, WFMT_4BIT_DQ = 0, 1, 2
NUM_PHASES = 28


class LoraError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("f", ctypes.c_int32), ("r", ctypes.c_int32),
                ("eps", ctypes.c_float), ("scale", ctypes.c_float), ("wfmt", ctypes.c_int32),
                ("qblock", ctypes.c_int32), ("residual", ctypes.c_int32)]


WEIGHT_FIELDS = ("Wg", "Wu", "Wd", "Qg", "Qu", "Qd", "absmax_g", "absmax_u", "absmax_d", "codebook",
                 "absmax8_g", "absmax8_u", "absmax8_d", "scale2_g", "scale2_u", "scale2_d")


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


class Adapters(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")]


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd", "dw")]


class CtxLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("rstd", "H", "G", "U", "Act", "P", "Pd", "total")] + \
               [("rp", ctypes.c_int32)]


class QkvDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("nq", ctypes.c_int32), ("nkv", ctypes.c_int32),
                ("r", ctypes.c_int32), ("eps", ctypes.c_float), ("scale", ctypes.c_float)]


class QkvWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("Wq", "Wk", "Wv")]


class QkvAdapters(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("Aq", "Bq", "Ak", "Bk", "Av", "Bv")]


class QkvGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dAq", "dBq", "dAk", "dBk", "dAv", "dBv")]


class QkvCtxLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("rstd", "H", "P", "total")] + [("rp", ctypes.c_int32)]


class ODims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("n_in", ctypes.c_int32), ("n_out", ctypes.c_int32), ("r", ctypes.c_int32),
                ("scale", ctypes.c_float)]


class CeDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("V", ctypes.c_int32), ("vocab_chunk", ctypes.c_int32),
                ("reduction", ctypes.c_int32)]


CE_MEAN, CE_SUM = 0, 1


def header_functions() -> list[str]:
    """Names of the functions include/lora_mlp.h declares."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(lora_\w+)\s*\(", txt, flags=re.M)


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m lora_fine_tuning_rmsnorm_b200.build` "
                          "(the LoRA-MLP path has no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    sig = {
        "lora_mlp_ctx_layout_get": [ctypes.POINTER(Dims), ctypes.POINTER(CtxLayout)],
        "lora_mlp_workspace_bytes": [ctypes.POINTER(Dims), ctypes.POINTER(ctypes.c_size_t)],
        "lora_mlp_fwd": [ctypes.POINTER(Dims), vp, vp, ctypes.POINTER(Weights), ctypes.POINTER(Adapters), vp, vp,
                         vp, vp],
        "lora_mlp_bwd": [ctypes.POINTER(Dims), vp, vp, vp, ctypes.POINTER(Weights), ctypes.POINTER(Adapters), vp,
                         vp, ctypes.POINTER(Grads), vp, vp],
        "lora_rmsnorm_fwd": [i64, i32, f32, vp, vp, vp, vp, vp],
        "lora_rmsnorm_bwd": [i64, i32, vp, vp, vp, vp, vp, vp],
        "lora_quantize_4bit": [vp, i64, i32, vp, vp, vp, vp],
        "lora_quantize_absmax8": [vp, i64, i32, vp, vp, vp],
        "lora_merge_weights": [i64, i64, i32, f32, vp, vp, vp, vp, vp],
        "lora_qkv_ctx_layout_get": [ctypes.POINTER(QkvDims), ctypes.POINTER(QkvCtxLayout)],
        "lora_qkv_workspace_bytes": [ctypes.POINTER(QkvDims), ctypes.POINTER(ctypes.c_size_t)],
        "lora_qkv_fwd": [ctypes.POINTER(QkvDims), vp, vp, ctypes.POINTER(QkvWeights), ctypes.POINTER(QkvAdapters),
                         vp, vp, vp, vp, vp, vp],
        "lora_qkv_bwd": [ctypes.POINTER(QkvDims), vp, vp, vp, vp, vp, ctypes.POINTER(QkvWeights),
                         ctypes.POINTER(QkvAdapters), vp, vp, ctypes.POINTER(QkvGrads), vp, vp],
        "lora_gemm_bf16": [i64, i64, i64, vp, i32, vp, i32, vp, i32, vp],
        "lora_lowrank_proj_noalloc": [i64, i32, i32, f32, vp, vp, vp, vp],
        "lora_mlp_status": [vp, ctypes.POINTER(ctypes.c_int32), vp],
        "lora_o_ctx_bytes": [ctypes.POINTER(ODims), ctypes.POINTER(ctypes.c_size_t)],
        "lora_o_workspace_bytes": [ctypes.POINTER(ODims), ctypes.POINTER(ctypes.c_size_t)],
        "lora_o_fwd": [ctypes.POINTER(ODims), vp, vp, vp, vp, vp, vp, vp, vp],
        "lora_o_bwd": [ctypes.POINTER(ODims), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "lora_rope": [i64, i32, i32, i32, vp, i64, vp, vp, vp, vp, i32, vp],
        "lora_ce_workspace_bytes": [ctypes.POINTER(CeDims), ctypes.POINTER(ctypes.c_size_t)],
        "lora_ce_fwd": [ctypes.POINTER(CeDims), vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "lora_ce_bwd": [ctypes.POINTER(CeDims), vp, vp, vp, vp, vp, f32, vp, vp, vp],
        "lora_mlp_timing_enable": [i32],
        "lora_mlp_timing_collect": [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.lora_mlp_last_error.restype = ctypes.c_char_p
    L.lora_mlp_last_error.argtypes = []
    L.lora_mlp_phase_name.restype = ctypes.c_char_p
    L.lora_mlp_phase_name.argtypes = [i32]
    _lib = L
    return L


def _check(rc: int):
    if rc != LORA_OK:
        raise LoraError(rc, lib().lora_mlp_last_error().decode())


def _p(t):
    """Device (or host) address of a tensor, or None."""
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_dims(T, d, f, r, eps=1e-6, scale=1.0, wfmt=WFMT_BF16, qblock=64, residual=False) -> Dims:
    return Dims(T, d, f, r, eps, scale, wfmt, qblock, int(bool(residual)))


def ctx_layout(dims: Dims) -> CtxLayout:
    out = CtxLayout()
    _check(lib().lora_mlp_ctx_layout_get(ctypes.byref(dims), ctypes.byref(out)))
    return out


def workspace_bytes(dims: Dims) -> int:
    out = ctypes.c_size_t()
    _check(lib().lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)))
    return out.value


def alloc_ctx(dims: Dims, device="cuda"):
    import torch
    return torch.empty(ctx_layout(dims).total, dtype=torch.uint8, device=device)


def alloc_workspace(dims: Dims, device="cuda"):
    import torch
    return torch.empty(workspace_bytes(dims), dtype=torch.uint8, device=device)


def ctx_views(dims: Dims, ctx):
    """Typed views of the saved context (rstd, H, G, U, Act, P, Pd) for inspection."""
    import torch
    L = ctx_layout(dims)
    T, d, f, rp = dims.T, dims.d, dims.f, L.rp

    def v(off, n, dt, shape):
        nbytes = n * (4 if dt == torch.float32 else 2)
        return ctx[off:off + nbytes].view(dt).view(*shape)
    return dict(rstd=v(L.rstd, T, torch.float32, (T,)), H=v(L.H, T * d, torch.bfloat16, (T, d)),
                G=v(L.G, T * f, torch.bfloat16, (T, f)), U=v(L.U, T * f, torch.bfloat16, (T, f)),
                Act=v(L.Act, T * f, torch.bfloat16, (T, f)), P=v(L.P, T * 2 * rp, torch.bfloat16, (T, 2 * rp)),
                Pd=v(L.Pd, T * rp, torch.bfloat16, (T, rp)))


def make_weights(**tensors) -> Weights:
    """Weights struct from tensors named as its fields (the others NULL)."""
    unknown = set(tensors) - set(WEIGHT_FIELDS)
    if unknown:
        raise TypeError(f"unknown weight fields {sorted(unknown)}")
    return Weights(*[_p(tensors.get(n)) for n in WEIGHT_FIELDS])


def make_adapters(Ag, Bg, Au, Bu, Ad, Bd) -> Adapters:
    return Adapters(*[_p(t) for t in (Ag, Bg, Au, Bu, Ad, Bd)])


def make_grads(dAg, dBg, dAu, dBu, dAd, dBd, dw=None) -> Grads:
    """dw (fp32 [d]) only for a trainable norm weight; None leaves it uncomputed."""
    return Grads(*[_p(t) for t in (dAg, dBg, dAu, dBu, dAd, dBd, dw)])


def merge_weights(W, A, B, scale, out=None, stream=None):
    """Wm = bf16(W + scale * B A) (W [rows x cols], A [r x cols], B [rows x r], bf16 on the
    device); `out` may be W itself (in place)."""
    import torch
    rows, cols = W.shape
    r = A.shape[0]
    out = torch.empty_like(W) if out is None else out
    _check(lib().lora_merge_weights(rows, cols, r, float(scale), _p(W), _p(A), _p(B), _p(out), _stream(stream)))
    return out


def lora_mlp_fwd(dims: Dims, X, rms_w, weights: Weights, adapters: Adapters, Y, ctx, workspace, stream=None):
    _check(lib().lora_mlp_fwd(ctypes.byref(dims), _p(X), _p(rms_w), ctypes.byref(weights),
                              ctypes.byref(adapters), _p(Y), _p(ctx), _p(workspace), _stream(stream)))


def lora_mlp_bwd(dims: Dims, dY, X, rms_w, weights: Weights, adapters: Adapters, ctx, dX, grads: Grads,
                 workspace, stream=None):
    _check(lib().lora_mlp_bwd(ctypes.byref(dims), _p(dY), _p(X), _p(rms_w), ctypes.byref(weights),
                              ctypes.byref(adapters), _p(ctx), _p(dX), ctypes.byref(grads), _p(workspace),
                              _stream(stream)))


def lora_rmsnorm_fwd(X, w, H, rstd, eps, stream=None):
    T, d = X.shape
    _check(lib().lora_rmsnorm_fwd(T, d, eps, _p(X), _p(w), _p(H), _p(rstd), _stream(stream)))


def lora_rmsnorm_bwd(dH, X, w, rstd, dX, stream=None):
    T, d = X.shape
    _check(lib().lora_rmsnorm_bwd(T, d, _p(dH), _p(X), _p(w), _p(rstd), _p(dX), _stream(stream)))


def lora_quantize_4bit(W, codebook, codes, absmax, block=64, stream=None):
    _check(lib().lora_quantize_4bit(_p(W), W.numel(), block, _p(codebook), _p(codes), _p(absmax),
                                    _stream(stream)))


def lora_quantize_absmax8(absmax, codes8, scale2, block2=256, stream=None):
    """Double quantisation of the 4-bit block constants: absmax fp32 -> codes8 uint8, scale2 fp32."""
    _check(lib().lora_quantize_absmax8(_p(absmax), absmax.numel(), block2, _p(codes8), _p(scale2),
                                       _stream(stream)))


GEMM_CTA_PAIR = 1
GEMM_TEST_NO_LOADS = 2


def lora_gemm_bf16(A, a_mn, B, b_mn, C, pair=False, stream=None, test_no_loads=False):
    """C = A' B'^T (see lora_gemm_bf16 in the header).  test_no_loads exercises the
    bounded-wait failure path: nothing is copied, the kernel's waits run out."""
    M, N = C.shape
    K = A.shape[0] if a_mn else A.shape[1]
    flags = (GEMM_CTA_PAIR if pair else 0) | (GEMM_TEST_NO_LOADS if test_no_loads else 0)
    _check(lib().lora_gemm_bf16(M, N, K, _p(A), int(a_mn), _p(B), int(b_mn), _p(C), flags, _stream(stream)))


def status(workspace=None, stream=None) -> int:
    """Bounded-wait status code of the last call that used `workspace` (None: the last
    workspace-less call in this context); 0 = every wait completed.  Synchronises."""
    code = ctypes.c_int32(0)
    rc = lib().lora_mlp_status(_p(workspace), ctypes.byref(code), _stream(stream))
    if rc not in (LORA_OK, -5):
        _check(rc)
    return code.value


def lora_lowrank_proj_noalloc(X, A, P, scale, stream=None):
    """P[T x rp] = scale * X A^T using the library's fixed device scratch (no allocation)."""
    T, K = X.shape
    r = A.shape[0]
    _check(lib().lora_lowrank_proj_noalloc(T, K, r, scale, _p(X), _p(A), _p(P), _stream(stream)))


def timing_enable(on: bool = True):
    _check(lib().lora_mlp_timing_enable(1 if on else 0))


def timing_collect() -> dict:
    ms = (ctypes.c_double * NUM_PHASES)()
    n = (ctypes.c_int64 * NUM_PHASES)()
    _check(lib().lora_mlp_timing_collect(ms, n))
    out = {}
    for i in range(NUM_PHASES):
        if n[i]:
            out[lib().lora_mlp_phase_name(i).decode()] = (ms[i], n[i])
    return out


# ------------------------------------------------------------------ Q/K/V projections
def qkv_dims(T, d, nq, nkv, r, eps=1e-6, scale=1.0) -> QkvDims:
    return QkvDims(T, d, nq, nkv, r, eps, scale)


def qkv_ctx_layout(dims: QkvDims) -> QkvCtxLayout:
    out = QkvCtxLayout()
    _check(lib().lora_qkv_ctx_layout_get(ctypes.byref(dims), ctypes.byref(out)))
    return out


def qkv_workspace_bytes(dims: QkvDims) -> int:
    out = ctypes.c_size_t()
    _check(lib().lora_qkv_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)))
    return out.value


def lora_qkv_fwd(dims: QkvDims, X, rms_w, weights: QkvWeights, adapters: QkvAdapters, Q, K, V, ctx, workspace,
                 stream=None):
    _check(lib().lora_qkv_fwd(ctypes.byref(dims), _p(X), _p(rms_w), ctypes.byref(weights), ctypes.byref(adapters),
                              _p(Q), _p(K), _p(V), _p(ctx), _p(workspace), _stream(stream)))


def lora_qkv_bwd(dims: QkvDims, dQ, dK, dV, X, rms_w, weights: QkvWeights, adapters: QkvAdapters, ctx, dX,
                 grads: QkvGrads, workspace, stream=None):
    _check(lib().lora_qkv_bwd(ctypes.byref(dims), _p(dQ), _p(dK), _p(dV), _p(X), _p(rms_w), ctypes.byref(weights),
                              ctypes.byref(adapters), _p(ctx), _p(dX), ctypes.byref(grads), _p(workspace),
                              _stream(stream)))


# ------------------------------------------------------------------ o_proj LoRA linear
def o_dims(T, n_in, n_out, r, scale=1.0) -> ODims:
    return ODims(T, n_in, n_out, r, scale)


def o_ctx_bytes(dims: ODims) -> int:
    out = ctypes.c_size_t()
    _check(lib().lora_o_ctx_bytes(ctypes.byref(dims), ctypes.byref(out)))
    return out.value


def o_workspace_bytes(dims: ODims) -> int:
    out = ctypes.c_size_t()
    _check(lib().lora_o_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)))
    return out.value


def lora_o_fwd(dims: ODims, X, Wo, Ao, Bo, Y, ctx, workspace, stream=None):
    _check(lib().lora_o_fwd(ctypes.byref(dims), _p(X), _p(Wo), _p(Ao), _p(Bo), _p(Y), _p(ctx), _p(workspace),
                            _stream(stream)))


def lora_o_bwd(dims: ODims, dY, X, Wo, Ao, Bo, ctx, dX, dAo, dBo, workspace, stream=None):
    _check(lib().lora_o_bwd(ctypes.byref(dims), _p(dY), _p(X), _p(Wo), _p(Ao), _p(Bo), _p(ctx), _p(dX), _p(dAo),
                            _p(dBo), _p(workspace), _stream(stream)))


# ------------------------------------------------------------------ RoPE
def lora_rope(Q, K, pos, cos, sin, hd, backward=False, stream=None):
    """Rotate Q [T x hq hd] and K [T x hk hd] (bf16, in place) at positions pos [T] int32
    with the fp32 tables cos, sin [n_pos x hd/2]; backward applies the inverse rotation."""
    T = pos.shape[0]
    hq = 0 if Q is None else Q.shape[1] // hd
    hk = 0 if K is None else K.shape[1] // hd
    _check(lib().lora_rope(T, hq, hk, hd, _p(pos), cos.shape[0], _p(cos), _p(sin), _p(Q), _p(K),
                           1 if backward else 0, _stream(stream)))


# ------------------------------------------------------------------ LM-head cross-entropy
def ce_dims(T, d, V, vocab_chunk=0, reduction=CE_MEAN) -> CeDims:
    return CeDims(T, d, V, vocab_chunk, reduction)


def ce_workspace_bytes(dims: CeDims) -> int:
    out = ctypes.c_size_t()
    _check(lib().lora_ce_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)))
    return out.value


def lora_ce_fwd(dims: CeDims, H, W, labels, loss_rows, lse, loss, n_valid, workspace, stream=None):
    _check(lib().lora_ce_fwd(ctypes.byref(dims), _p(H), _p(W), _p(labels), _p(loss_rows), _p(lse), _p(loss),
                             _p(n_valid), _p(workspace), _stream(stream)))


def lora_ce_bwd(dims: CeDims, H, W, labels, lse, n_valid, dloss, dH, workspace, stream=None):
    _check(lib().lora_ce_bwd(ctypes.byref(dims), _p(H), _p(W), _p(labels), _p(lse), _p(n_valid), float(dloss),
                             _p(dH), _p(workspace), _stream(stream)))
