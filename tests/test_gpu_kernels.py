"""GPU parity of the building blocks through the C ABI: the tcgen05 GEMM core (all
operand majors, ragged sizes), the RMSNorm row kernels, the 4-bit quantiser."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import ops, synth
from lora_fine_tuning_rmsnorm_b200.runner import bf16_tensor
from oracle import lora_mlp_ref as ref
from oracle import quant4_ref as q4
from tests.parity import assert_close, to_np

pytestmark = pytest.mark.gpu


def rand_bf16(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    bits = synth.f32_to_bf16_bits((scale * rng.standard_normal(shape)).astype(np.float32))
    return bits, synth.bf16_bits_to_f64(bits)


GEMM_SIZES = [(128, 256, 64), (200, 136, 344), (64, 64, 8), (384, 512, 1024), (136, 72, 200), (520, 264, 128)]


@pytest.mark.parametrize("pair", [False, True], ids=["1cta", "pair"])
@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("M,N,K", GEMM_SIZES)
def test_gemm_core(cuda_ok, M, N, K, a_mn, b_mn, pair):
    if pair and a_mn:
        pytest.skip("CTA pairs take a K-major A operand")
    Ab, Af = rand_bf16((K, M) if a_mn else (M, K), 1 + M + K)
    Bb, Bf = rand_bf16((K, N) if b_mn else (N, K), 2 + N + K)
    A = bf16_tensor(Ab)
    B = bf16_tensor(Bb)
    C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ops.lora_gemm_bf16(A, a_mn, B, b_mn, C, pair=pair)
    torch.cuda.synchronize()
    Am = Af.T if a_mn else Af
    Bm = Bf.T if b_mn else Bf
    R = Am @ Bm.T
    out = to_np(C)
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out, R, rtol=0, atol=1e-5 * np.abs(R).max() * max(1.0, np.sqrt(K / 64)))


@pytest.mark.parametrize("T,d", [(64, 128), (77, 2048), (130, 4096), (5, 8), (33, 16384)])
def test_rmsnorm_fwd_bwd(cuda_ok, T, d):
    Xb, X = rand_bf16((T, d), 3, 1.0)
    wb = synth.f32_to_bf16_bits((1 + 0.1 * np.random.default_rng(4).standard_normal(d)).astype(np.float32))
    w = synth.bf16_bits_to_f64(wb)
    eps = 1e-6
    Xt, wt = bf16_tensor(Xb), bf16_tensor(wb)
    H = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    rstd = torch.empty(T, dtype=torch.float32, device="cuda")
    ops.lora_rmsnorm_fwd(Xt, wt, H, rstd, eps)
    Hr, rr = ref.rmsnorm_fwd(X, w, eps)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_np(rstd), rr, rtol=2e-6)
    assert_close("H", to_np(H), Hr, rel_fro=4e-3, max_rel=8e-3)
    dH = torch.from_numpy(np.random.default_rng(5).standard_normal((T, d)).astype(np.float32)).cuda()
    dX = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    ops.lora_rmsnorm_bwd(dH, Xt, wt, rstd, dX)
    torch.cuda.synchronize()
    dXr = ref.rmsnorm_bwd(to_np(dH), X, w, rr)
    assert_close("dX", to_np(dX), dXr, rel_fro=4e-3, max_rel=8e-3)


def test_quantize_bit_exact(cuda_ok):
    rng = np.random.default_rng(7)
    f, d = 344, 128
    W = (0.02 * rng.standard_normal((f, d))).astype(np.float32)
    W[3, :64] = 0.0                        # an all-zero block
    W[5, 64:] = -0.0
    code = q4.codebook16()
    m = q4.midpoints(code)
    W[7, 0] = 0.125                        # block absmax (exact in bf16)
    W[7, 1:16] = (0.125 * m.astype(np.float64)).astype(np.float32)  # near the midpoints
    Wb = synth.f32_to_bf16_bits(W)
    Wf = synth.bf16_bits_to_f64(Wb)
    idx_ref, am_ref = q4.quantize(Wf, code)
    Wt = bf16_tensor(Wb)
    cb = torch.from_numpy(code).cuda()
    codes = torch.empty(f * d // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(f * d // 64, dtype=torch.float32, device="cuda")
    ops.lora_quantize_4bit(Wt, cb, codes, absmax)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(absmax.cpu().numpy(), am_ref)
    np.testing.assert_array_equal(q4.unpack(codes.cpu().numpy()), idx_ref)
