"""Device-side set-up of one LoRA-MLP problem: upload seeded bf16 inputs, allocate
outputs / saved context / workspace with torch, and call the C ABI.  Marshalling
only; the arithmetic runs in liblora_mlp.so."""
from __future__ import annotations

import numpy as np
import torch

from . import ops, synth

ADAPTERS = ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")
GRADS = ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd")


def bf16_tensor(bits: np.ndarray, device="cuda", pin=False) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    if device == "cpu":
        return t.pin_memory() if pin else t
    return t.to(device)


class Problem:
    """All device buffers of one fwd+bwd step for a Shape."""

    def __init__(self, shape: synth.Shape, bits: dict | None = None, seed: int = synth.BASE_SEED,
                 device="cuda", residual: bool = False, norm_grad: bool = False):
        self.shape = s = shape
        self.device = device
        bits = bits if bits is not None else synth.make_inputs_bits(s, seed)
        self.t = {k: bf16_tensor(v, device) for k, v in bits.items()}
        self.dims = ops.make_dims(s.T, s.d, s.f, s.r, eps=s.eps, scale=s.scale, residual=residual)
        self.weights = ops.make_weights(Wg=self.t["Wg"], Wu=self.t["Wu"], Wd=self.t["Wd"])
        self.adapters = ops.make_adapters(*(self.t[k] for k in ADAPTERS))
        self.Y = torch.empty(s.T, s.d, dtype=torch.bfloat16, device=device)
        self.dX = torch.empty(s.T, s.d, dtype=torch.bfloat16, device=device)
        shapes = {"dAg": (s.r, s.d), "dBg": (s.f, s.r), "dAu": (s.r, s.d), "dBu": (s.f, s.r),
                  "dAd": (s.r, s.f), "dBd": (s.d, s.r)}
        self.g = {k: torch.empty(*shapes[k], dtype=torch.float32, device=device) for k in GRADS}
        self.dw = torch.empty(s.d, dtype=torch.float32, device=device) if norm_grad else None
        self.grads = ops.make_grads(*(self.g[k] for k in GRADS), dw=self.dw)
        self.ctx = ops.alloc_ctx(self.dims, device)
        self.ws = ops.alloc_workspace(self.dims, device)

    def use_4bit(self, codebook, drop_bf16: bool = True, double_quant: bool = False):
        """Quantise the frozen Wg, Wu, Wd to 4-bit blockwise codes on the GPU (one-off
        set-up, lora_quantize_4bit) and switch the weights to them.  `codebook` is the
        16-entry fp32 code table (an input of the method).  double_quant also quantises
        the block constants (lora_quantize_absmax8) and switches to that format."""
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
        if double_quant:
            a8, s2 = {}, {}
            for k in ("g", "u", "d"):
                n = absmax[k].numel()
                a8[k] = torch.empty(n, dtype=torch.uint8, device=self.device)
                s2[k] = torch.empty((n + 255) // 256, dtype=torch.float32, device=self.device)
                ops.lora_quantize_absmax8(absmax[k], a8[k], s2[k])
            self.dims.wfmt = ops.WFMT_4BIT_DQ
            self.dq = (a8, s2)
            # this format's workspace also holds the expanded constants: size it anew
            self.ws = ops.alloc_workspace(self.dims, self.device)
            self.weights = ops.make_weights(Qg=codes["g"], Qu=codes["u"], Qd=codes["d"], codebook=cb,
                                            absmax8_g=a8["g"], absmax8_u=a8["u"], absmax8_d=a8["d"],
                                            scale2_g=s2["g"], scale2_u=s2["u"], scale2_d=s2["d"])
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


class HostPipeline:
    """Training-step driver for inputs and results in pinned HOST memory.

    Every step copies its X and dY host -> device, runs lora_mlp_fwd + lora_mlp_bwd,
    and copies Y, dX and the packed adapter gradients device -> host.  The copies are
    double-buffered, one stream per direction (`xs` inputs in, `ss` results out, so the
    two directions of the host link run at the same time): step i's results go back and
    step i+2's inputs come in while step i+1 computes.  Events order the buffers: a step
    computes once its inputs are in (`ready`) and the results of the step before it in the
    same buffer are out (`stored`); its buffer is refilled once it has computed (`done`).
    `reduce` (optional) is called on the packed gradient buffer on the compute stream after
    each backward (the data-parallel all-reduce).
    """

    def __init__(self, pb: "Problem", hX: torch.Tensor, hdY: torch.Tensor, reduce=None):
        from . import dist as ldist
        s = pb.shape
        self.pb, self.hX, self.hdY, self.reduce = pb, hX, hdY, reduce
        dev = pb.Y.device
        self.cs = torch.cuda.current_stream(dev)
        self.xs = torch.cuda.Stream(dev)
        self.ss = torch.cuda.Stream(dev)
        self.bufs = []
        for _ in range(2):
            flat, views = ldist.flat_grads(s.d, s.f, s.r, device=dev)
            self.bufs.append(dict(X=torch.empty_like(hX, device=dev), dY=torch.empty_like(hdY, device=dev),
                                  Y=torch.empty(s.T, s.d, dtype=torch.bfloat16, device=dev),
                                  dX=torch.empty(s.T, s.d, dtype=torch.bfloat16, device=dev), flat=flat,
                                  grads=ops.make_grads(*(views[k] for k in GRADS)),
                                  ready=torch.cuda.Event(), done=torch.cuda.Event(), stored=torch.cuda.Event()))
        self.hY = torch.empty(s.T, s.d, dtype=torch.bfloat16, pin_memory=True)
        self.hdX = torch.empty(s.T, s.d, dtype=torch.bfloat16, pin_memory=True)
        self.hflat = torch.empty(self.bufs[0]["flat"].numel(), dtype=torch.float32, pin_memory=True)
        self.h2d_bytes = hX.numel() * hX.element_size() + hdY.numel() * hdY.element_size()
        self.d2h_bytes = 2 * self.hY.numel() * 2 + self.hflat.numel() * 4

    def _load(self, b):
        with torch.cuda.stream(self.xs):
            b["X"].copy_(self.hX, non_blocking=True)
            b["dY"].copy_(self.hdY, non_blocking=True)
            b["ready"].record(self.xs)

    def start(self):
        for b in self.bufs:
            self._load(b)

    def step(self, i: int, n_steps: int | None = None):
        """Run step i; with n_steps given, inputs are not prefetched past the last step."""
        pb, b = self.pb, self.bufs[i % 2]
        self.cs.wait_event(b["ready"])
        self.cs.wait_event(b["stored"])  # step i - 2's results have left this buffer
        ops.lora_mlp_fwd(pb.dims, b["X"], pb.t["w"], pb.weights, pb.adapters, b["Y"], pb.ctx, pb.ws, self.cs)
        ops.lora_mlp_bwd(pb.dims, b["dY"], b["X"], pb.t["w"], pb.weights, pb.adapters, pb.ctx, b["dX"],
                         b["grads"], pb.ws, self.cs)
        if self.reduce is not None:
            self.reduce(b["flat"])
        b["done"].record(self.cs)
        self.ss.wait_event(b["done"])
        with torch.cuda.stream(self.ss):
            self.hY.copy_(b["Y"], non_blocking=True)
            self.hdX.copy_(b["dX"], non_blocking=True)
            self.hflat.copy_(b["flat"], non_blocking=True)
            b["stored"].record(self.ss)
        if n_steps is None or i + 2 < n_steps:
            self.xs.wait_event(b["done"])
            self._load(b)  # inputs of step i + 2 (after this step's compute has read them)

    def finish(self):
        """Make the input stream wait for the results' copies: an event recorded on `xs`
        afterwards completes after every step's copies and compute."""
        self.xs.wait_stream(self.ss)


QKV_GRADS = ("dAq", "dBq", "dAk", "dBk", "dAv", "dBv")


class QkvProblem:
    """All device buffers of one Q/K/V-projection fwd+bwd step for a QkvShape."""

    def __init__(self, shape: synth.QkvShape, bits: dict | None = None, seed: int = synth.BASE_SEED,
                 device="cuda"):
        self.shape = s = shape
        bits = bits if bits is not None else synth.make_qkv_inputs_bits(s, seed)
        self.t = {k: bf16_tensor(v, device) for k, v in bits.items()}
        self.dims = ops.qkv_dims(s.T, s.d, s.nq, s.nkv, s.r, eps=s.eps, scale=s.scale)
        self.weights = ops.QkvWeights(*(ops._p(self.t[k]) for k in ("Wq", "Wk", "Wv")))
        self.adapters = ops.QkvAdapters(*(ops._p(self.t[k]) for k in ("Aq", "Bq", "Ak", "Bk", "Av", "Bv")))
        n = {"q": s.nq, "k": s.nkv, "v": s.nkv}
        self.out = {k: torch.empty(s.T, n[k.lower()], dtype=torch.bfloat16, device=device) for k in ("Q", "K", "V")}
        self.dX = torch.empty(s.T, s.d, dtype=torch.bfloat16, device=device)
        shapes = {"dAq": (s.r, s.d), "dBq": (s.nq, s.r), "dAk": (s.r, s.d), "dBk": (s.nkv, s.r),
                  "dAv": (s.r, s.d), "dBv": (s.nkv, s.r)}
        self.g = {k: torch.empty(*shapes[k], dtype=torch.float32, device=device) for k in QKV_GRADS}
        self.grads = ops.QkvGrads(*(ops._p(self.g[k]) for k in QKV_GRADS))
        L = ops.qkv_ctx_layout(self.dims)
        self.ctx = torch.empty(L.total, dtype=torch.uint8, device=device)
        self.ws = torch.empty(ops.qkv_workspace_bytes(self.dims), dtype=torch.uint8, device=device)

    def forward(self, stream=None):
        ops.lora_qkv_fwd(self.dims, self.t["X"], self.t["w"], self.weights, self.adapters, self.out["Q"],
                         self.out["K"], self.out["V"], self.ctx, self.ws, stream)

    def backward(self, stream=None):
        ops.lora_qkv_bwd(self.dims, self.t["dQ"], self.t["dK"], self.t["dV"], self.t["X"], self.t["w"],
                         self.weights, self.adapters, self.ctx, self.dX, self.grads, self.ws, stream)

    def step(self, stream=None):
        self.forward(stream)
        self.backward(stream)


class OProblem:
    """All device buffers of one o_proj LoRA-linear fwd+bwd step for an OShape."""

    def __init__(self, shape: synth.OShape, bits: dict | None = None, seed: int = synth.BASE_SEED, device="cuda"):
        self.shape = s = shape
        bits = bits if bits is not None else synth.make_o_inputs_bits(s, seed)
        self.t = {k: bf16_tensor(v, device) for k, v in bits.items()}
        self.dims = ops.o_dims(s.T, s.n_in, s.n_out, s.r, scale=s.scale)
        self.Y = torch.empty(s.T, s.n_out, dtype=torch.bfloat16, device=device)
        self.dX = torch.empty(s.T, s.n_in, dtype=torch.bfloat16, device=device)
        self.dAo = torch.empty(s.r, s.n_in, dtype=torch.float32, device=device)
        self.dBo = torch.empty(s.n_out, s.r, dtype=torch.float32, device=device)
        self.ctx = torch.empty(ops.o_ctx_bytes(self.dims), dtype=torch.uint8, device=device)
        self.ws = torch.empty(ops.o_workspace_bytes(self.dims), dtype=torch.uint8, device=device)

    def forward(self, stream=None):
        t = self.t
        ops.lora_o_fwd(self.dims, t["X"], t["Wo"], t["Ao"], t["Bo"], self.Y, self.ctx, self.ws, stream)

    def backward(self, stream=None):
        t = self.t
        ops.lora_o_bwd(self.dims, t["dY"], t["X"], t["Wo"], t["Ao"], t["Bo"], self.ctx, self.dX, self.dAo, self.dBo,
                       self.ws, stream)

    def step(self, stream=None):
        self.forward(stream)
        self.backward(stream)


class RopeProblem:
    """Device buffers of one RoPE forward (Q, K in place) + backward (dQ, dK in place)."""

    def __init__(self, shape: synth.RopeShape, data: dict | None = None, seed: int = synth.BASE_SEED,
                 device="cuda"):
        self.shape = s = shape
        data = data if data is not None else synth.make_rope_inputs(s, seed)
        self.t = {k: bf16_tensor(data[k], device) for k in ("Q", "K", "dQ", "dK")}
        self.pos = torch.from_numpy(np.ascontiguousarray(data["pos"], dtype=np.int32)).to(device)
        self.cos = torch.from_numpy(np.ascontiguousarray(data["cos"], dtype=np.float32)).to(device)
        self.sin = torch.from_numpy(np.ascontiguousarray(data["sin"], dtype=np.float32)).to(device)

    def forward(self, stream=None):
        ops.lora_rope(self.t["Q"], self.t["K"], self.pos, self.cos, self.sin, self.shape.hd, False, stream)

    def backward(self, stream=None):
        ops.lora_rope(self.t["dQ"], self.t["dK"], self.pos, self.cos, self.sin, self.shape.hd, True, stream)

    def step(self, stream=None):
        self.forward(stream)
        self.backward(stream)


class CeProblem:
    """Device buffers of one fused LM-head cross-entropy forward + backward for a CeShape."""

    def __init__(self, shape: synth.CeShape, data: dict | None = None, seed: int = synth.BASE_SEED, device="cuda",
                 vocab_chunk: int = 0, reduction: int = ops.CE_MEAN, dloss: float = 1.0):
        self.shape = s = shape
        data = data if data is not None else synth.make_ce_inputs(s, seed)
        self.H = bf16_tensor(data["H"], device)
        self.W = bf16_tensor(data["W"], device)
        self.labels = torch.from_numpy(np.ascontiguousarray(data["labels"], dtype=np.int32)).to(device)
        self.dims = ops.ce_dims(s.T, s.d, s.V, vocab_chunk, reduction)
        self.dloss = dloss
        self.loss_rows = torch.empty(s.T, dtype=torch.float32, device=device)
        self.lse = torch.empty(s.T, dtype=torch.float32, device=device)
        self.stats = torch.zeros(4, dtype=torch.int32, device=device)   # [0] loss (fp32 bits), [1] n_valid
        self.loss = self.stats[0:1].view(torch.float32)
        self.n_valid = self.stats[1:2]
        self.dH = torch.empty(s.T, s.d, dtype=torch.float32, device=device)
        self.ws = torch.empty(ops.ce_workspace_bytes(self.dims), dtype=torch.uint8, device=device)

    def forward(self, stream=None):
        ops.lora_ce_fwd(self.dims, self.H, self.W, self.labels, self.loss_rows, self.lse, self.loss, self.n_valid,
                        self.ws, stream)

    def backward(self, stream=None):
        ops.lora_ce_bwd(self.dims, self.H, self.W, self.labels, self.lse, self.n_valid, self.dloss, self.dH, self.ws,
                        stream)

    def step(self, stream=None):
        self.forward(stream)
        self.backward(stream)
