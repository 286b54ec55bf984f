"""The LoRA-MLP workloads: shapes only (tokens T, hidden d, intermediate f, rank r).

The shapes stand in for the pages' fine-tuning workloads: Llama-3-8B / Llama-3.2-1B
LoRA/QLoRA SFT at sequence 2048 and batch 4 ("Unsloth提速秘诀：Triton内核如何加速反向传播",
§4.1; "Unsloth 深度实战", §3.2), with alpha = 16 and eps = 1e-6.
"""
from .synth import CeShape, OShape, QkvShape, RopeShape, Shape

TINY = Shape(T=64, d=128, f=344, r=8, alpha=16.0)            # batch 2 x seq 32
LLAMA32_1B = Shape(T=8192, d=2048, f=8192, r=16, alpha=16.0)  # batch 4 x seq 2048
LLAMA3_8B = Shape(T=8192, d=4096, f=14336, r=16, alpha=16.0)  # batch 4 x seq 2048

# rank / length sweep at the 8B width (batch 1, long rows); alpha = 16 throughout
SWEEP = [Shape(T=T, d=4096, f=14336, r=r, alpha=16.0)
         for r in (8, 16, 32, 64, 128) for T in (512, 2048, 8192, 32768)]

QBLOCK = 64  # 4-bit blockwise quantisation block size


def algorithmic_flops(s: Shape) -> float:
    """Dense 12*T*d*f (6 fwd + 6 bwd, frozen W gets no gradient) + LoRA 18*T*r*(d+f)."""
    return 12.0 * s.T * s.d * s.f + 18.0 * s.T * s.r * (s.d + s.f)


# attention Q/K/V projections of the same 8B model: 32 query heads and 8 key/value heads
# of 128 (grouped-query attention), batch 4 x seq 2048
QKV_8B = QkvShape(T=8192, d=4096, nq=4096, nkv=1024, r=16, alpha=16.0)


def qkv_algorithmic_flops(s: QkvShape) -> float:
    """Dense 4*T*d*N with N = nq + 2 nkv (forward and input gradient; frozen W gets no
    gradient) + LoRA 2*T*r*(9 d + 3 N) (P, P B^T; Q, the dH term, dA, dB)."""
    N = s.nq + 2 * s.nkv
    return 4.0 * s.T * s.d * N + 2.0 * s.T * s.r * (9 * s.d + 3 * N)


# the same model's attention output projection (32 heads x 128 -> hidden 4096) and the
# rotary embedding of its 32 query / 8 key heads (head dim 128, Llama-3 rotary base
# 500000), batch 4 x seq 2048
O_8B = OShape(T=8192, n_in=4096, n_out=4096, r=16, alpha=16.0)
ROPE_8B = RopeShape(T=8192, hq=32, hk=8, hd=128, seq_len=2048, base=500000.0)


def o_algorithmic_flops(s: OShape) -> float:
    """Dense 4*T*n_in*n_out (Y and dX; frozen Wo gets no gradient) + LoRA
    2*T*r*(3 n_in + 3 n_out) (P, P Bo^T, Q, Q Ao, dAo, dBo)."""
    return 4.0 * s.T * s.n_in * s.n_out + 6.0 * s.T * s.r * (s.n_in + s.n_out)


def rope_bytes(s: RopeShape) -> float:
    """HBM bytes of one RoPE launch: Q and K read and written once (bf16)."""
    return 4.0 * s.T * (s.hq + s.hk) * s.hd


# the same model's LM-head cross-entropy: hidden 4096, vocabulary 128256, batch 4 x seq 2048
CE_8B = CeShape(T=8192, d=4096, V=128256)


def ce_algorithmic_flops(s: CeShape) -> float:
    """Logits in the forward (2 T d V), recomputed logits and dH in the backward (4 T d V)."""
    return 6.0 * s.T * s.d * s.V
