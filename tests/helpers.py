"""Shared test helpers: configuration dicts and small brute-force references."""
import numpy as np

from synth import MODELS, ModelShape


def oracle_cfg(m: ModelShape, k_max: int) -> dict:
    return dict(hidden=m.hidden, n_q_heads=m.n_q_heads, n_kv_heads=m.n_kv_heads,
                head_dim=m.head_dim, inter=m.inter, vocab=m.vocab, n_prelude=m.n_prelude,
                n_core=m.n_core, n_coda=m.n_coda, k_max=k_max, rope_base=m.rope_base,
                rms_eps=m.rms_eps, qk_norm=m.qk_norm, mask_id=m.mask_id)


def small_shape(**kw) -> ModelShape:
    base = dict(name="pin", hidden=32, n_q_heads=4, n_kv_heads=2, head_dim=8, inter=48,
                vocab=64, n_prelude=1, n_core=2, n_coda=1, weight_dtype="fp32")
    base.update(kw)
    return ModelShape(**base)
