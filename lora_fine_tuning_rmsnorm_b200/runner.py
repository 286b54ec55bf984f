"""Device-side set-up of one LoRA-MLP problem: upload seeded bf16 inputs, allocate
outputs / saved context / workspace with torch, and call the C ABI.  Marshalling
only; the arithmetic runs in liblora_mlp.so."""
from __future__ import annotations

import numpy as np
import torch

from . import ops, synth

ADAPTERS = ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")
GRADS = ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd")


def load_codebook() -> list:
    """The 16-entry 4-bit codebook written by tests/golden/make_codebook.py."""
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests", "golden",
                        "codebook16.json")
    with open(path) as fh:
        return [float.fromhex(h) for h in json.load(fh)["codebook_f32_hex"]]


def bf16_tensor(bits: np.ndarray, device="cuda", pin=False) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    if device == "cpu":
        return t.pin_memory() if pin else t
    return t.to(device)


class Problem:
    """All device buffers of one fwd+bwd step for a Shape."""

    def __init__(self, shape: synth.Shape, bits: dict | None = None, seed: int = synth.BASE_SEED,
                 device="cuda"):
        self.shape = s = shape
        self.device = device
        bits = bits if bits is not None else synth.make_inputs_bits(s, seed)
        self.t = {k: bf16_tensor(v, device) for k, v in bits.items()}
        self.dims = ops.make_dims(s.T, s.d, s.f, s.r, eps=s.eps, scale=s.scale)
        self.weights = ops.make_weights(Wg=self.t["Wg"], Wu=self.t["Wu"], Wd=self.t["Wd"])
        self.adapters = ops.make_adapters(*(self.t[k] for k in ADAPTERS))
        self.Y = torch.empty(s.T, s.d, dtype=torch.bfloat16, device=device)
        self.dX = torch.empty(s.T, s.d, dtype=torch.bfloat16, device=device)
        shapes = {"dAg": (s.r, s.d), "dBg": (s.f, s.r), "dAu": (s.r, s.d), "dBu": (s.f, s.r),
                  "dAd": (s.r, s.f), "dBd": (s.d, s.r)}
        self.g = {k: torch.empty(*shapes[k], dtype=torch.float32, device=device) for k in GRADS}
        self.grads = ops.make_grads(*(self.g[k] for k in GRADS))
        self.ctx = ops.alloc_ctx(self.dims, device)
        self.ws = ops.alloc_workspace(self.dims, device)

    def use_4bit(self, codebook, drop_bf16: bool = True):
        """Quantise the frozen Wg, Wu, Wd to 4-bit blockwise codes on the GPU (one-off
        set-up, lora_quantize_4bit) and switch the weights to them.  `codebook` is the
        16-entry fp32 code table (an input of the method)."""
        cb = torch.as_tensor(np.asarray(codebook, dtype=np.float32)).to(self.device)
        codes, absmax = {}, {}
        for k, name in (("g", "Wg"), ("u", "Wu"), ("d", "Wd")):
            W = self.t[name]
            codes[k] = torch.empty(W.numel() // 2, dtype=torch.uint8, device=self.device)
            absmax[k] = torch.empty(W.numel() // 64, dtype=torch.float32, device=self.device)
            ops.lora_quantize_4bit(W, cb, codes[k], absmax[k])
        self.dims.wfmt = ops.WFMT_4BIT
        self.dims.qblock = 64
        self.q4 = (codes, absmax, cb)
        self.weights = ops.make_weights(Qg=codes["g"], Qu=codes["u"], Qd=codes["d"], absmax_g=absmax["g"],
                                        absmax_u=absmax["u"], absmax_d=absmax["d"], codebook=cb)
        if drop_bf16:  # the bf16 copies are no longer needed on the device
            for name in ("Wg", "Wu", "Wd"):
                self.t[name] = None

    def forward(self, X=None, stream=None):
        ops.lora_mlp_fwd(self.dims, self.t["X"] if X is None else X, self.t["w"], self.weights, self.adapters,
                         self.Y, self.ctx, self.ws, stream)

    def backward(self, dY=None, X=None, stream=None):
        ops.lora_mlp_bwd(self.dims, self.t["dY"] if dY is None else dY, self.t["X"] if X is None else X,
                         self.t["w"], self.weights, self.adapters, self.ctx, self.dX, self.grads, self.ws, stream)

    def step(self, stream=None):
        self.forward(stream=stream)
        self.backward(stream=stream)

    def saved(self) -> dict:
        return ops.ctx_views(self.dims, self.ctx)
