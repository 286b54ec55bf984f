"""GPU parity of the fused LM-head cross-entropy (lora_ce_fwd / lora_ce_bwd through the C
ABI) against the fp64 oracle: per-token loss and logsumexp, the reduced loss and the kept
count, and dH, at ragged small shapes (vocabularies that are not tile multiples, several
vocabulary chunks in the backward, ignored and out-of-range labels, both reductions) and
at the Llama-3-8B head (d = 4096, V = 128256, T = 8192) on sampled rows."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, ops, synth
from lora_fine_tuning_rmsnorm_b200.runner import CeProblem
from oracle import ce_ref
from tests.parity import assert_close, to_np

pytestmark = pytest.mark.gpu

CASES = [  # (T, d, V, vocab_chunk, reduction)
    (64, 128, 344, 0, ops.CE_MEAN),
    (200, 136, 1000, 0, ops.CE_MEAN),
    (300, 256, 4096, 1024, ops.CE_MEAN),    # four vocabulary chunks in the backward
    (129, 64, 520, 256, ops.CE_SUM),        # three chunks, the last one ragged
    (37, 8, 24, 0, ops.CE_MEAN),            # d = 8: one partial K block
]


def run(shape, data, chunk, reduction, dloss=1.0):
    pb = CeProblem(shape, data, vocab_chunk=chunk, reduction=reduction, dloss=dloss)
    pb.dH.fill_(float("nan"))
    pb.step()
    torch.cuda.synchronize()
    assert ops.status(pb.ws) == 0
    return pb


@pytest.mark.parametrize("T,d,V,chunk,reduction", CASES, ids=[f"T{c[0]}_d{c[1]}_V{c[2]}_c{c[3]}_r{c[4]}" for c in CASES])
def test_ce_parity_small(cuda_ok, T, d, V, chunk, reduction):
    shape = synth.CeShape(T=T, d=d, V=V)
    data = synth.make_ce_inputs(shape)
    data["labels"][3] = V + 5                # out of range: left out like the ignore index
    data["labels"][T - 1] = V - 1            # the last vocabulary column
    pb = run(shape, data, chunk, reduction, dloss=0.75)
    H, W = synth.bf16_bits_to_f64(data["H"]), synth.bf16_bits_to_f64(data["W"])
    red = "mean" if reduction == ops.CE_MEAN else "sum"
    R = ce_ref.forward(H, W, data["labels"], red)
    assert int(pb.n_valid.item()) == R["n_valid"]
    np.testing.assert_allclose(to_np(pb.lse), R["lse"], rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(to_np(pb.loss_rows), R["loss_rows"], rtol=0, atol=2e-5 * max(1.0, np.abs(R["lse"]).max()))
    assert abs(float(pb.loss.item()) - R["loss"]) <= 1e-5 * max(1.0, abs(R["loss"]))
    dH = ce_ref.backward(H, W, data["labels"], 0.75, red)
    assert_close("dH", to_np(pb.dH), dH)
    ok = ce_ref.valid(data["labels"], V)
    assert torch.all(pb.dH[torch.from_numpy(~ok).cuda()] == 0)


def test_ce_no_kept_token(cuda_ok):
    shape = synth.CeShape(T=50, d=64, V=200)
    data = synth.make_ce_inputs(shape)
    data["labels"][:] = synth.IGNORE_INDEX
    pb = run(shape, data, 0, ops.CE_MEAN)
    assert int(pb.n_valid.item()) == 0 and float(pb.loss.item()) == 0.0
    assert torch.all(pb.loss_rows == 0) and torch.all(pb.dH == 0)


@pytest.mark.slow
def test_ce_parity_llama3_8b_sampled_rows(cuda_ok):
    shape = configs.CE_8B
    data = synth.make_ce_inputs(shape)
    pb = run(shape, data, 0, ops.CE_MEAN)
    labels = data["labels"]
    ok = ce_ref.valid(labels, shape.V)
    n = int(ok.sum())
    assert int(pb.n_valid.item()) == n
    rows_all = to_np(pb.loss_rows)
    # the reduced loss is the mean of the per-token losses over the kept tokens
    assert abs(float(pb.loss.item()) - rows_all[ok].mean()) <= 1e-5 * abs(rows_all[ok].mean())
    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 4095, 8191], rng.integers(0, shape.T, 40),
                                     np.nonzero(~ok)[0][:3]]))
    H, W = synth.bf16_bits_to_f64(data["H"]), synth.bf16_bits_to_f64(data["W"])
    R = ce_ref.rows_fwd_bwd(H, W, labels, rows, n)
    np.testing.assert_allclose(to_np(pb.lse)[rows], R["lse"], rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(rows_all[rows], R["loss_rows"], rtol=0, atol=5e-4)
    assert_close("dH rows", to_np(pb.dH)[rows], R["dH"])
