"""Parameter-shape tables of the benchmark workloads.

The pages evaluate FlashOptim on ResNet-50 (ImageNet), GPT-2 pretraining
and Llama-3.1-8B finetuning.  No dataset, checkpoint or model is needed
for the optimizer step: only the list of parameter tensors matters, so the
workloads below are those models' parameter shapes with synthetic values
(see ``workloads.gen`` for the generator).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import numpy as np

from . import gen


@dataclass(frozen=True)
class TensorSpec:
    name: str
    shape: Tuple[int, ...]
    init: str            # "normal" | "const"
    value: float         # sigma for "normal", the constant for "const"

    @property
    def numel(self) -> int:
        return int(np.prod(self.shape)) if self.shape else 1


@dataclass
class Workload:
    name: str
    tensors: List[TensorSpec]
    optimizer: str                 # "adamw" | "sgdm"
    hparams: Dict[str, float]
    w_dtype: str = "bf16"
    grad_dtype: str = "bf16"
    ecc_bits: int = 8
    grad_dist: str = "normal"      # "normal" | "normal_outliers" | "student_t3"
    grad_scale: float = 1e-3
    seed: int = 0
    warm_steps: int = 0
    description: str = ""
    extra: Dict[str, object] = field(default_factory=dict)

    @property
    def numel(self) -> int:
        return sum(t.numel for t in self.tensors)

    # ---- host generation (random access by element index) ----
    def master_values(self, ti: int, idx: np.ndarray) -> np.ndarray:
        spec = self.tensors[ti]
        idx = np.asarray(idx, np.int64)
        if spec.init == "const":
            return np.full(idx.shape, spec.value, np.float32)
        key = gen.stream_key(self.seed, ti, 0, gen.KIND_MASTER)
        return gen.normal(key, idx, spec.value)

    def grad_values(self, ti: int, step: int, idx: np.ndarray) -> np.ndarray:
        """float32 gradient values (before the cast to the grad dtype)."""
        idx = np.asarray(idx, np.int64)
        key = gen.stream_key(self.seed, ti, step, gen.KIND_GRAD)
        if self.grad_dist == "student_t3":
            return gen.student_t3(key, idx, self.grad_scale)
        z = gen.normal(key, idx, self.grad_scale)
        if self.grad_dist == "normal_outliers":
            ko = gen.stream_key(self.seed, ti, step, gen.KIND_OUTLIER)
            z = np.where(gen.outlier_mask(ko, idx), z * np.float32(100.0), z)
        return z

    def grad_bits(self, ti: int, step: int, idx: np.ndarray) -> np.ndarray:
        return gen.to_16bit(self.grad_values(ti, step, idx), self.grad_dtype)


ADAMW_HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
SGDM_HP = dict(lr=0.1, momentum=0.9, dampening=0.0, weight_decay=1e-4, nesterov=0)


def flat_1m() -> Workload:
    return Workload(
        name="flat-1M",
        tensors=[TensorSpec("flat", (1048576,), "normal", 0.02)],
        optimizer="adamw", hparams=dict(ADAMW_HP), grad_dist="normal", grad_scale=1e-3,
        warm_steps=0, extra=dict(steps=10),
        description="one flat group of 1,048,576 params, 10 AdamW steps from zero states")


def gpt2_small() -> Workload:
    d, v, ctx, L = 768, 50257, 1024, 12
    ts = [TensorSpec("wte", (v, d), "normal", 0.02), TensorSpec("wpe", (ctx, d), "normal", 0.02)]
    for i in range(L):
        p = f"h.{i}."
        ts += [
            TensorSpec(p + "ln_1.weight", (d,), "const", 1.0),
            TensorSpec(p + "ln_1.bias", (d,), "const", 0.0),
            TensorSpec(p + "attn.c_attn.weight", (d, 3 * d), "normal", 0.02),
            TensorSpec(p + "attn.c_attn.bias", (3 * d,), "const", 0.0),
            TensorSpec(p + "attn.c_proj.weight", (d, d), "normal", 0.02),
            TensorSpec(p + "attn.c_proj.bias", (d,), "const", 0.0),
            TensorSpec(p + "ln_2.weight", (d,), "const", 1.0),
            TensorSpec(p + "ln_2.bias", (d,), "const", 0.0),
            TensorSpec(p + "mlp.c_fc.weight", (d, 4 * d), "normal", 0.02),
            TensorSpec(p + "mlp.c_fc.bias", (4 * d,), "const", 0.0),
            TensorSpec(p + "mlp.c_proj.weight", (4 * d, d), "normal", 0.02),
            TensorSpec(p + "mlp.c_proj.bias", (d,), "const", 0.0),
        ]
    ts += [TensorSpec("ln_f.weight", (d,), "const", 1.0), TensorSpec("ln_f.bias", (d,), "const", 0.0)]
    return Workload(
        name="gpt2-small-124M", tensors=ts, optimizer="adamw", hparams=dict(ADAMW_HP),
        grad_dist="normal_outliers", grad_scale=1e-3, warm_steps=100,
        description="GPT-2-small parameter list (148 tensors), 1% gradient outliers x100, "
                    "one multi-tensor AdamW step after 100 warm steps")


def gpt2_small_sgdm() -> Workload:
    """The GPT-2-small parameter list stepped by SGD-momentum with fp16 + 8-bit
    ECC masters (the ResNet-50 recipe's optimizer and formats): an SGD-momentum
    case whose 1.26 GB per step is ten times the L2, for profiler captures."""
    w = gpt2_small()
    return Workload(
        name="gpt2-small-124M-sgdm", tensors=w.tensors, optimizer="sgdm", hparams=dict(SGDM_HP),
        w_dtype="fp16", grad_dtype="fp16", grad_dist="normal", grad_scale=1e-2, warm_steps=1,
        description="GPT-2-small parameter list (148 tensors), fp16 + 8-bit ECC masters, "
                    "SGD momentum 0.9")


def _conv(name, cout, cin, k):
    return TensorSpec(name, (cout, cin, k, k), "normal", math.sqrt(2.0 / (cin * k * k)))


def resnet50() -> Workload:
    ts: List[TensorSpec] = [_conv("conv1.weight", 64, 3, 7),
                            TensorSpec("bn1.weight", (64,), "const", 1.0),
                            TensorSpec("bn1.bias", (64,), "const", 0.0)]
    cin = 64
    for li, (width, blocks) in enumerate([(64, 3), (128, 4), (256, 6), (512, 3)], start=1):
        cout = width * 4
        for b in range(blocks):
            p = f"layer{li}.{b}."
            ts += [_conv(p + "conv1.weight", width, cin, 1),
                   TensorSpec(p + "bn1.weight", (width,), "const", 1.0),
                   TensorSpec(p + "bn1.bias", (width,), "const", 0.0),
                   _conv(p + "conv2.weight", width, width, 3),
                   TensorSpec(p + "bn2.weight", (width,), "const", 1.0),
                   TensorSpec(p + "bn2.bias", (width,), "const", 0.0),
                   _conv(p + "conv3.weight", cout, width, 1),
                   TensorSpec(p + "bn3.weight", (cout,), "const", 1.0),
                   TensorSpec(p + "bn3.bias", (cout,), "const", 0.0)]
            if b == 0:
                ts += [_conv(p + "downsample.0.weight", cout, cin, 1),
                       TensorSpec(p + "downsample.1.weight", (cout,), "const", 1.0),
                       TensorSpec(p + "downsample.1.bias", (cout,), "const", 0.0)]
            cin = cout
    ts += [TensorSpec("fc.weight", (1000, 2048), "normal", math.sqrt(2.0 / 2048)),
           TensorSpec("fc.bias", (1000,), "const", 0.0)]
    return Workload(
        name="resnet50-25.6M", tensors=ts, optimizer="sgdm", hparams=dict(SGDM_HP),
        w_dtype="fp16", grad_dtype="fp16", grad_dist="normal", grad_scale=1e-2, warm_steps=1,
        description="ResNet-50 parameter list (161 tensors), fp16 + 8-bit ECC masters, "
                    "SGD momentum 0.9")


def llama31_8b(order: str = "forward", ecc_bits: int = 8) -> Workload:
    d, v, L, ffn, kv = 4096, 128256, 32, 14336, 1024
    ts = [TensorSpec("embed_tokens.weight", (v, d), "normal", 0.02)]
    for i in range(L):
        p = f"layers.{i}."
        ts += [
            TensorSpec(p + "input_layernorm.weight", (d,), "const", 1.0),
            TensorSpec(p + "self_attn.q_proj.weight", (d, d), "normal", 0.02),
            TensorSpec(p + "self_attn.k_proj.weight", (kv, d), "normal", 0.02),
            TensorSpec(p + "self_attn.v_proj.weight", (kv, d), "normal", 0.02),
            TensorSpec(p + "self_attn.o_proj.weight", (d, d), "normal", 0.02),
            TensorSpec(p + "post_attention_layernorm.weight", (d,), "const", 1.0),
            TensorSpec(p + "mlp.gate_proj.weight", (ffn, d), "normal", 0.02),
            TensorSpec(p + "mlp.up_proj.weight", (ffn, d), "normal", 0.02),
            TensorSpec(p + "mlp.down_proj.weight", (d, ffn), "normal", 0.02),
        ]
    ts += [TensorSpec("norm.weight", (d,), "const", 1.0),
           TensorSpec("lm_head.weight", (v, d), "normal", 0.02)]
    name = "llama3.1-8b" + ("" if ecc_bits == 8 else "-ecc16")
    wl = Workload(
        name=name, tensors=ts, optimizer="adamw", hparams=dict(ADAMW_HP),
        ecc_bits=ecc_bits, grad_dist="student_t3", grad_scale=1e-4, warm_steps=0,
        description="Llama-3.1-8B parameter list (291 tensors), Student-t(3) x 1e-4 gradients, "
                    "one AdamW step from zero states")
    if order == "release":
        wl.name += "-release"
        wl.extra["launch"] = "per-tensor, reverse layer order"
    return wl


def llama31_layers(n_layers: int = 2, ecc_bits: int = 8) -> Workload:
    """The first decoder layers of the Llama-3.1-8B list (same shapes, values
    and hyper-parameters as in the full list): a case of a few GB, far above
    the L2, for profiler captures of the full-size kernel."""
    full = llama31_8b()
    per_layer = 9
    ts = full.tensors[1:1 + per_layer * n_layers]
    return Workload(
        name=f"llama3.1-8b-{n_layers}layers" + ("" if ecc_bits == 8 else "-ecc16"), tensors=ts, optimizer="adamw",
        hparams=dict(ADAMW_HP), ecc_bits=ecc_bits, grad_dist="student_t3", grad_scale=1e-4, warm_steps=0,
        description=f"decoder layers 0..{n_layers - 1} of the Llama-3.1-8B parameter list"
                    + ("" if ecc_bits == 8 else ", 16-bit ECC"))


CONFIGS = {
    "flat-1M": flat_1m,
    "gpt2-small-124M": gpt2_small,
    "gpt2-small-124M-sgdm": gpt2_small_sgdm,
    "resnet50-25.6M": resnet50,
    "llama3.1-8b": llama31_8b,
    "llama3.1-8b-2layers": llama31_layers,
}


def workload(name: str) -> Workload:
    if name == "llama3.1-8b-release":
        return llama31_8b("release")
    if name == "llama3.1-8b-ecc16":
        return llama31_8b(ecc_bits=16)
    if name == "llama3.1-8b-2layers-ecc16":
        return llama31_layers(2, ecc_bits=16)
    return CONFIGS[name]()
