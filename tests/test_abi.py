"""The C-ABI library: it loads, exports every function include/lora_mlp.h declares,
and rejects bad arguments on the host with the documented codes (no GPU needed:
validation happens before any CUDA call)."""
import ctypes

import pytest

from lora_fine_tuning_rmsnorm_b200 import build, ops


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.lib()


def test_exports_every_declared_symbol(L):
    names = ops.header_functions()
    assert {"lora_mlp_fwd", "lora_mlp_bwd", "lora_rmsnorm_fwd", "lora_rmsnorm_bwd", "lora_quantize_4bit",
            "lora_gemm_bf16", "lora_mlp_ctx_layout_get", "lora_mlp_workspace_bytes",
            "lora_mlp_last_error"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_layout_and_workspace_sizes(L):
    dims = ops.make_dims(8192, 4096, 14336, 16)
    lay = ops.ctx_layout(dims)
    assert lay.rp == 16
    T, d, f = 8192, 4096, 14336
    assert lay.H - lay.rstd >= T * 4 and lay.G - lay.H >= T * d * 2
    assert lay.total >= T * 4 + T * d * 2 + 3 * T * f * 2 + 3 * T * 16 * 2
    for off in (lay.rstd, lay.H, lay.G, lay.U, lay.Act, lay.P, lay.Pd):
        assert off % 256 == 0
    ws = ops.workspace_bytes(dims)
    assert ws >= T * d * 4 + 2 * T * f * 2
    assert ops.ctx_layout(ops.make_dims(64, 128, 344, 8)).rp == 16


@pytest.mark.parametrize("T,d,f,r,code", [
    (0, 128, 344, 8, ops.ERRORS and -1),
    (64, 0, 344, 8, -1),
    (64, 130, 344, 8, -2),
    (64, 128, 340, 8, -2),
    (64, 128, 344, 12, -2),
    (64, 128, 344, 136, -3),
    (64, 70000, 344, 8, -3),
])
def test_bad_dims_rejected(L, T, d, f, r, code):
    dims = ops.make_dims(T, d, f, r)
    out = ctypes.c_size_t()
    rc = L.lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out))
    assert rc == code
    assert len(L.lora_mlp_last_error()) > 0


def test_null_and_misaligned_pointers_rejected(L):
    dims = ops.make_dims(64, 128, 344, 8)
    w = ops.Weights()
    a = ops.Adapters()
    rc = L.lora_mlp_fwd(ctypes.byref(dims), None, None, ctypes.byref(w), ctypes.byref(a), None, None, None, None)
    assert rc == -1
    assert b"NULL" in L.lora_mlp_last_error()
    bad = ctypes.c_void_p(0x1001)
    good = ctypes.c_void_p(0x1000)
    rc = L.lora_rmsnorm_fwd(64, 128, 1e-6, bad, good, good, good, None)
    assert rc == -2
    rc = L.lora_rmsnorm_fwd(64, 129, 1e-6, good, good, good, good, None)
    assert rc == -1
    rc = L.lora_quantize_4bit(good, 100, 64, good, good, good, None)
    assert rc == -1
    rc = L.lora_quantize_4bit(good, 128, 32, good, good, good, None)
    assert rc == -3
    rc = L.lora_gemm_bf16(64, 60, 64, good, 0, good, 0, good, 0, None)
    assert rc == -2
    g = ops.Grads()
    rc = L.lora_mlp_bwd(ctypes.byref(dims), good, good, good, ctypes.byref(w), ctypes.byref(a), good, good,
                        ctypes.byref(g), good, None)
    assert rc == -1


def test_4bit_dims_rules(L):
    dims = ops.make_dims(64, 256, 344, 8, wfmt=ops.WFMT_4BIT)
    out = ctypes.c_size_t()
    assert L.lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)) == -3   # f % 256 != 0
    dims = ops.make_dims(64, 128, 512, 8, wfmt=ops.WFMT_4BIT)
    assert L.lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)) == -3   # d % 256 != 0
    dims = ops.make_dims(64, 256, 512, 8, wfmt=ops.WFMT_4BIT, qblock=32)
    assert L.lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)) == -3
    dims = ops.make_dims(64, 256, 512, 8, wfmt=ops.WFMT_4BIT)
    assert L.lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)) == 0


def test_phase_names(L):
    names = [L.lora_mlp_phase_name(i).decode() for i in range(ops.NUM_PHASES)]
    assert "gemm_gate_up_swiglu" in names and "rmsnorm_fwd" in names
    assert L.lora_mlp_phase_name(99) == b"invalid"


def test_residual_flag_and_dw_pointer_checked(L):
    dims = ops.make_dims(64, 128, 344, 8)
    dims.residual = 2
    out = ctypes.c_size_t()
    assert L.lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)) == -1
    dims.residual = 1
    assert L.lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)) == 0
    good = ctypes.c_void_p(0x1000)
    w = ops.Weights(*([0x1000] * 3))
    a = ops.Adapters(*([0x1000] * 6))
    g = ops.Grads(*([0x1000] * 6 + [0x1004]))   # dw given but not 16-byte aligned
    rc = L.lora_mlp_bwd(ctypes.byref(dims), good, good, good, ctypes.byref(w), ctypes.byref(a), good, good,
                        ctypes.byref(g), good, None)
    assert rc == -2


def test_merge_weights_argument_checks(L):
    good = ctypes.c_void_p(0x1000)
    assert L.lora_merge_weights(0, 64, 8, 1.0, good, good, good, good, None) == -1          # rows
    assert L.lora_merge_weights(16, 60, 8, 1.0, good, good, good, good, None) == -1         # cols % 8
    assert L.lora_merge_weights(16, 64, 300, 1.0, good, good, good, good, None) == -3       # r > 256
    assert L.lora_merge_weights(16, 64, 8, float("inf"), good, good, good, good, None) == -1
    assert L.lora_merge_weights(16, 64, 8, 1.0, ctypes.c_void_p(0x1008), good, good, good, None) == -2
    assert L.lora_merge_weights(16, 64, 8, 1.0, good, good, ctypes.c_void_p(0x1001), good, None) == -2


def test_qkv_layout_and_argument_checks(L):
    dims = ops.qkv_dims(8192, 4096, 4096, 1024, 16)
    lay = ops.qkv_ctx_layout(dims)
    assert lay.rp == 16
    for off in (lay.rstd, lay.H, lay.P):
        assert off % 256 == 0
    assert lay.total >= 8192 * 4 + 8192 * 4096 * 2 + 8192 * 48 * 2
    assert ops.qkv_workspace_bytes(dims) >= 8192 * 4096 * 4 + 8192 * 48 * 2
    out = ctypes.c_size_t()
    for bad, code in (((64, 128, 128, 60, 8), -2), ((64, 128, 0, 64, 8), -1), ((64, 128, 128, 64, 136), -3),
                      ((0, 128, 128, 64, 8), -1)):
        assert L.lora_qkv_workspace_bytes(ctypes.byref(ops.qkv_dims(*bad)), ctypes.byref(out)) == code, bad
    w, a, g = ops.QkvWeights(), ops.QkvAdapters(), ops.QkvGrads()
    good = ctypes.c_void_p(0x1000)
    rc = L.lora_qkv_fwd(ctypes.byref(ops.qkv_dims(64, 128, 128, 64, 8)), good, good, ctypes.byref(w), ctypes.byref(a),
                        good, good, good, good, good, None)
    assert rc == -1 and b"NULL" in L.lora_mlp_last_error()
    rc = L.lora_qkv_bwd(ctypes.byref(ops.qkv_dims(64, 128, 128, 64, 8)), good, good, good, good, good,
                        ctypes.byref(w), ctypes.byref(a), good, good, ctypes.byref(g), good, None)
    assert rc == -1


def test_gemm_flags_and_status_argument_checks(L):
    good = ctypes.c_void_p(0x1000)
    assert L.lora_gemm_bf16(64, 64, 64, good, 0, good, 0, good, 4, None) == -1        # unknown flag
    assert L.lora_gemm_bf16(64, 64, 64, good, 0, good, 0, good, 3, None) == -1        # test flag + pair
    assert b"single-CTA" in L.lora_mlp_last_error()
    code = ctypes.c_int32(0)
    assert L.lora_mlp_status(ctypes.c_void_p(0x1004), ctypes.byref(code), None) == -2  # misaligned workspace


def test_o_proj_and_rope_argument_checks(L):
    out = ctypes.c_size_t()
    good = ctypes.c_void_p(0x1000)
    for bad, code in (((64, 130, 64, 8), -2), ((0, 128, 64, 8), -1), ((64, 128, 64, 136), -3), ((64, 128, 0, 8), -1)):
        assert L.lora_o_workspace_bytes(ctypes.byref(ops.o_dims(*bad)), ctypes.byref(out)) == code, bad
    dims = ops.o_dims(8192, 4096, 4096, 16)
    assert ops.o_ctx_bytes(dims) >= 8192 * 16 * 2
    assert ops.o_workspace_bytes(dims) >= 256 + 8192 * 16 * 2
    assert L.lora_o_fwd(ctypes.byref(dims), good, None, good, good, good, good, good, None) == -1
    assert L.lora_o_bwd(ctypes.byref(dims), good, good, good, good, good, good, good, good, ctypes.c_void_p(0x1008),
                        good, None) == -2
    # rope: hd a multiple of 16, head counts, pointers
    assert L.lora_rope(16, 2, 1, 24, good, 16, good, good, good, good, 0, None) == -2
    assert L.lora_rope(16, 0, 0, 64, good, 16, good, good, good, good, 0, None) == -1
    assert L.lora_rope(16, 2, 1, 64, good, 16, good, good, good, good, 2, None) == -1
    assert L.lora_rope(16, 2, 1, 64, None, 16, good, good, good, good, 0, None) == -1
    assert L.lora_rope(16, 2, 1, 64, good, 16, good, good, good, None, 0, None) == -1   # K needed when hk > 0


def test_ce_argument_checks(L):
    out = ctypes.c_size_t()
    good = ctypes.c_void_p(0x1000)
    for bad, code in (((64, 130, 344), -2), ((64, 128, 340), -2), ((0, 128, 344), -1), ((64, 4, 344), -1)):
        assert L.lora_ce_workspace_bytes(ctypes.byref(ops.ce_dims(*bad)), ctypes.byref(out)) == code, bad
    assert L.lora_ce_workspace_bytes(ctypes.byref(ops.ce_dims(64, 128, 344, vocab_chunk=100)), ctypes.byref(out)) == -1
    assert L.lora_ce_workspace_bytes(ctypes.byref(ops.ce_dims(64, 128, 344, reduction=2)), ctypes.byref(out)) == -1
    big = ops.ce_workspace_bytes(ops.ce_dims(8192, 4096, 128256))
    assert big >= 8192 * 32768 * 2                         # one vocabulary chunk of dZ (bf16)
    assert ops.ce_workspace_bytes(ops.ce_dims(8192, 4096, 128256, vocab_chunk=8192)) < big
    dims = ops.ce_dims(64, 128, 344)
    assert L.lora_ce_fwd(ctypes.byref(dims), good, good, good, good, good, ctypes.c_void_p(0x1002), good, good,
                         None) == -2                        # loss not 4-byte aligned
    assert L.lora_ce_fwd(ctypes.byref(dims), good, None, good, good, good, good, good, good, None) == -1
    assert L.lora_ce_bwd(ctypes.byref(dims), good, good, good, good, good, float("nan"), good, good, None) == -1


def test_double_quant_argument_checks(L):
    good = ctypes.c_void_p(0x1000)
    assert L.lora_quantize_absmax8(good, 1000, 128, good, good, None) == -3        # block2 must be 256
    assert L.lora_quantize_absmax8(good, 0, 256, good, good, None) == -1
    assert L.lora_quantize_absmax8(good, 1000, 256, good, ctypes.c_void_p(0x1004), None) == -2
    dims = ops.make_dims(64, 256, 512, 8, wfmt=ops.WFMT_4BIT_DQ)
    out = ctypes.c_size_t()
    assert L.lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)) == 0
    plain = ops.workspace_bytes(ops.make_dims(64, 256, 512, 8, wfmt=ops.WFMT_4BIT))
    assert out.value >= plain + 3 * (256 * 512 // 64) * 4           # the expanded constants
    dims = ops.make_dims(64, 256, 344, 8, wfmt=ops.WFMT_4BIT_DQ)
    assert L.lora_mlp_workspace_bytes(ctypes.byref(dims), ctypes.byref(out)) == -3   # f % 256
    # the double-quantised format needs its own constant arrays, not absmax
    dims = ops.make_dims(64, 256, 512, 8, wfmt=ops.WFMT_4BIT_DQ)
    w = ops.make_weights(Qg=None)
    for f in ("Qg", "Qu", "Qd", "codebook", "absmax_g", "absmax_u", "absmax_d"):
        setattr(w, f, 0x1000)
    a = ops.Adapters(*([0x1000] * 6))
    rc = L.lora_mlp_fwd(ctypes.byref(dims), good, good, ctypes.byref(w), ctypes.byref(a), good, good, good, None)
    assert rc == -1 and b"NULL" in L.lora_mlp_last_error()
