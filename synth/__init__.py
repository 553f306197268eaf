"""Seeded synthetic inputs for the ALoDLM denoising step.

This module holds shapes, workload presets and random-number generation only.
It computes nothing of the method: both the CPU oracle (through the tests) and the
CUDA library consume what it produces, and neither depends on the other.

Model shapes follow the Qwen3 conversions named by the paper digest "ALoDLM: Adaptively
Looped Diffusion Language Models" (section "Core method": 8B = Prelude layers [0,10),
Recurrent Core [10,26), Coda [26,36)), plus two small shapes that the oracle finishes in
seconds.  No trained weights or datasets are used here: weights are drawn
from seeded normals, prefix ids are uniform random ids, and the decoded block is all
[MASK], standing in for the GSM8K prompts the paper decodes with a 16-token window.

Weight scales (the paper gives none for random init):
  * every projection matrix and the embedding: N(0, 0.02)
  * RMSNorm gains 1, final-norm gain 4
  * LM head N(0, (3.2/sqrt(H))^2): logit std about 12.8 at every width, as in the tiny
    config (0.2 * 4 * sqrt(256))
  * ExitGate weight N(0, (0.02*sqrt(256/H))^2), bias -1
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class ModelShape:
    name: str
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    inter: int
    vocab: int
    n_prelude: int
    n_core: int
    n_coda: int
    rope_base: float = 1.0e6
    rms_eps: float = 1.0e-6
    qk_norm: int = 1
    weight_dtype: str = "bf16"  # storage type of the generated weights: "bf16" or "fp32"

    @property
    def n_layers(self) -> int:
        return self.n_prelude + self.n_core + self.n_coda

    @property
    def mask_id(self) -> int:
        return self.vocab - 1


MODELS: Dict[str, ModelShape] = {
    # hidden 256, 4q/2kv, hd 64, SwiGLU 688, vocab 2048, layers 1/2/1, fp32 weights
    "tiny": ModelShape("tiny", 256, 4, 2, 64, 688, 2048, 1, 2, 1, weight_dtype="fp32"),
    # several tiles with ragged tails everywhere: hidden 320 (2.5 x 128), GQA group 3,
    # head_dim 128, SwiGLU 880 (ragged k-tail), vocab 3001 (ragged vocab tile)
    "mid": ModelShape("mid", 320, 6, 2, 128, 880, 3001, 2, 3, 2),
    # Prelude 0 / Coda 0 special case: the whole stack loops
    "tiny_fullcore": ModelShape("tiny_fullcore", 256, 4, 2, 64, 688, 2048, 0, 2, 0, weight_dtype="fp32"),
    # narrow model with the Qwen3-8B attention geometry (32 q / 8 kv heads, head_dim 128):
    # kernel-level profiling of the step's attention and small kernels on a few-MB footprint
    "attn-probe": ModelShape("attn-probe", 256, 32, 8, 128, 256, 1024, 1, 1, 1),
    # the Qwen3-8B LM head and width with one layer per stage: profiling the fused readout on a
    # few GB of device memory
    "readout-probe": ModelShape("readout-probe", 4096, 32, 8, 128, 12288, 151936, 1, 1, 1),
    # Qwen3-1.7B shape, 28 layers split 8 / 12 / 8
    "qwen3-1.7b": ModelShape("qwen3-1.7b", 2048, 16, 8, 128, 6144, 151936, 8, 12, 8),
    # Qwen3-8B shape, 36 layers split 10 / 16 / 10
    "qwen3-8b": ModelShape("qwen3-8b", 4096, 32, 8, 128, 12288, 151936, 10, 16, 10),
}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    model: str
    batch: int
    prefix: int
    block: int
    k_max: int
    taus: tuple
    lambdas: tuple
    mixed_exit_depths: bool = False


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", "tiny", 1, 48, 16, 4, (0.1, 0.6, 0.9), (0.1, 0.9)),
    "mid": Workload("mid", "mid", 3, 75, 20, 5, (0.1, 0.6, 0.9), (0.1, 0.9)),
    "attn-probe-bs1": Workload("attn-probe-bs1", "attn-probe", 1, 1024, 32, 2, (0.6,), (0.5,)),
    "attn-probe-bs32": Workload("attn-probe-bs32", "attn-probe", 32, 2048, 64, 2, (0.6,), (0.5,)),
    # two and three 128-row query tiles per (sequence, KV head): the step attention's two-tile kernel
    "attn-probe-pq": Workload("attn-probe-pq", "attn-probe", 12, 160, 72, 3, (0.6,), (0.5,)),
    "readout-probe-bs1": Workload("readout-probe-bs1", "readout-probe", 1, 1024, 32, 2, (0.6,), (0.5,)),
    "qwen3-1.7b-bs1": Workload("qwen3-1.7b-bs1", "qwen3-1.7b", 1, 512, 32, 8, (0.6,), (0.5,)),
    "qwen3-8b-bs1": Workload("qwen3-8b-bs1", "qwen3-8b", 1, 1024, 32, 8, (0.6,), (0.5,)),
    "qwen3-8b-bs32": Workload("qwen3-8b-bs32", "qwen3-8b", 32, 2048, 64, 8, (0.1, 0.6, 0.9), (0.1, 0.9)),
    "qwen3-8b-long": Workload("qwen3-8b-long", "qwen3-8b", 8, 8192, 32, 12, (0.6,), (0.9,),
                              mixed_exit_depths=True),
}


# ----------------------------------------------------------------------------------
# weights
# ----------------------------------------------------------------------------------

LAYER_KEYS = ("attn_norm", "q", "k", "v", "o", "q_norm", "k_norm", "mlp_norm", "gate", "up", "down")
GLOBAL_KEYS = ("embed", "lm_head", "final_norm", "exit_w")


def layer_shapes(m: ModelShape) -> Dict[str, tuple]:
    H, hd = m.hidden, m.head_dim
    return {
        "attn_norm": (H,),
        "q": (m.n_q_heads * hd, H),
        "k": (m.n_kv_heads * hd, H),
        "v": (m.n_kv_heads * hd, H),
        "o": (H, m.n_q_heads * hd),
        "q_norm": (hd,),
        "k_norm": (hd,),
        "mlp_norm": (H,),
        "gate": (m.inter, H),
        "up": (m.inter, H),
        "down": (H, m.inter),
    }


def _tensor_seed(seed: int, index: int) -> int:
    return (int(seed) << 20) + int(index)


def _normal(shape, std: float, seed: int, index: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(_tensor_seed(seed, index))
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(std)


def make_weights(m: ModelShape, seed: int = 0, device: str = "cpu", only_layers: Optional[List[int]] = None,
                 with_globals: bool = True) -> dict:
    """Seeded random weights.

    Returns {"embed", "lm_head", "final_norm", "exit_w", "exit_b", "layers": [dict, ...]}.
    Matrices are torch tensors of dtype bfloat16 (weight_dtype "bf16") or float32;
    norm gains and the ExitGate weight are float32.  Tensor t of the canonical order is
    drawn from its own generator seeded with (seed << 20) + t, so one tensor can be
    regenerated alone.  On "cpu" the stream is identical on every machine; on "cuda" it is
    the CUDA generator's stream (used for the 1.7B/8B shapes, whose host copy is taken
    from the device tensors when needed).  ``only_layers``: generate just these layers (the
    others are None); ``with_globals=False`` leaves the embedding, LM head, final norm and
    ExitGate weight None; each generated tensor is the same as in the full draw.
    """
    H = m.hidden
    mat_dtype = torch.bfloat16 if m.weight_dtype == "bf16" else torch.float32
    out: dict = {}
    idx = 0

    def mat(shape, std, make=True):
        nonlocal idx
        t = _normal(shape, std, seed, idx, device).to(mat_dtype) if make else None
        idx += 1
        return t

    def vec(shape, value, make=True):
        nonlocal idx
        idx += 1
        return torch.full(shape, float(value), dtype=torch.float32, device=device) if make else None

    out["embed"] = mat((m.vocab, H), 0.02, with_globals)
    out["lm_head"] = mat((m.vocab, H), 3.2 / math.sqrt(H), with_globals)
    out["final_norm"] = vec((H,), 4.0, with_globals)
    idx_exit = idx
    out["exit_w"] = _normal((H,), 0.02 * math.sqrt(256.0 / H), seed, idx_exit, device) if with_globals else None
    idx += 1
    out["exit_b"] = -1.0
    layers: List[Optional[dict]] = []
    shapes = layer_shapes(m)
    for li in range(m.n_layers):
        make = only_layers is None or li in only_layers
        lw = {}
        for key in LAYER_KEYS:
            shp = shapes[key]
            if len(shp) == 1:
                lw[key] = vec(shp, 1.0, make)
            else:
                lw[key] = mat(shp, 0.02, make)
        layers.append(lw if make else None)
    out["layers"] = layers
    return out


def weights_to_numpy(w: dict, layers: Optional[List[int]] = None) -> dict:
    """Host float32 copy of (a subset of) the weights, for the oracle."""
    def cv(t):
        return t.detach().to(torch.float32).cpu().numpy()

    out = {k: cv(w[k]) for k in GLOBAL_KEYS}
    out["exit_b"] = float(w["exit_b"])
    sel = range(len(w["layers"])) if layers is None else layers
    out["layers"] = {i: {k: cv(v) for k, v in w["layers"][i].items()} for i in sel}
    if layers is None:
        out["layers"] = [out["layers"][i] for i in range(len(w["layers"]))]
    return out


# ----------------------------------------------------------------------------------
# inputs
# ----------------------------------------------------------------------------------

def make_prefix_ids(m: ModelShape, batch: int, prefix: int, seed: int = 1) -> np.ndarray:
    """Prefix ids uniform over [0, vocab-1): [MASK] (= vocab-1) never appears in a prefix."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, m.vocab - 1, size=(batch, prefix), dtype=np.int64).astype(np.int32)


def make_block_ids(m: ModelShape, batch: int, block: int, n_given: int = 0, seed: int = 3) -> np.ndarray:
    """Block ids: all [MASK], except n_given seeded positions per sequence holding real ids."""
    ids = np.full((batch, block), m.mask_id, dtype=np.int32)
    if n_given:
        rng = np.random.Generator(np.random.PCG64(seed))
        for b in range(batch):
            pos = rng.choice(block, size=n_given, replace=False)
            ids[b, pos] = rng.integers(0, m.vocab - 1, size=n_given)
    return ids


def make_exit_depths(batch: int, prefix: int, k_max: int, seed: int = 2) -> np.ndarray:
    """Per-prefix-position exit depths, uniform over 1..k_max."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(1, k_max + 1, size=(batch, prefix), dtype=np.int64).astype(np.int32)
