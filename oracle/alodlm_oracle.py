"""Oracle for one ALoDLM denoising step: a plain, slow CPU statement of the method.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference leg of ``bench.py`` may import or run this module.  The CUDA library never
does, and this module imports nothing of it.

Sources are the pages collected on ALoDLM.  Citations name the page and its section:

* [digest]  "ALoDLM: Adaptively Looped Diffusion Language Models" (paper digest page).
    - section "Core method" (核心方法): Prelude / Recurrent Core / Coda; each loop the
      Core updates the state, the Coda reads out r^(s); r^(s) feeds the LMHead
      (distribution, entropy commit H <= tau) and the ExitGate
      lambda = sigmoid(ExitGate(sg[r])); the loop ends once the mean cumulative halt of
      the unresolved positions reaches q, and s = K forces the exit.
    - same section, Eq. 3: h_i^(s) = Emb(y_i) for a committed position, else h~_i^(s).
    - section "Method steps" (方法步骤详情), Algorithm 1 steps (1)-(5).
    - section "Technical novelty" (技术新颖性): depth-aware KV cache (matching depth first,
      deepest available as fallback); the 8B path executes 10 + 4 x (16 + 10) = 114 layers.
    - section "Prerequisites" (前置知识), KV-cache paragraph: the same physical layer gives
      different KV at different loop depths.
    - section "Limitations" (局限与改进): L + (K-1) m = 84 logical KV buffers for the 8B.
    - section "Results" (实验结果): greedy decoding.
* [summary] tokendh.com lay summary: two heads (token guess, "think again?"), committed
  tokens become context, unresolved positions keep their internal state.

Where the pages are silent the oracle takes these readings (each is also a reading
of the CUDA library, stated in its header):

* Layers are pre-norm Qwen3 decoder layers: RMSNorm, QKV, per-head RMSNorm of q and k,
  rotate-half RoPE (base 1e6), softmax attention with grouped KV heads, output
  projection, residual; RMSNorm, SwiGLU MLP, residual.
* Prefill attention over the prefix is causal.  The block attends to every prefix
  position and to every block position (bidirectional); the prefix never sees the block.
* Positions: prefix 0..P-1, block P..P+N-1.
* The Coda KV of the prefix is one set, computed from each position's exit-depth state.
* Token choice is argmax (lowest id on ties); entropy is in nats over the full vocab.
* "Emb" is the input embedding, unscaled.  The ExitGate is Linear(H -> 1) with bias,
  applied to r^(s) (after the final RMSNorm).
* Two commit rules (they differ on the role of the halting threshold):
    PAPER      commit {i in U : H_i <= tau}; stop when U is empty, when the mean of a
               over the remaining U reaches q (``lam``), or at s = K; if nothing was
               committed in the whole step, commit the single lowest-entropy position
               of the last loop (lowest index on ties); the rest stay [MASK].
    PER_TOKEN  commit {i in U : H_i <= tau or a_i >= lam}, and all of U at s = K;
               stop when U is empty.
* a is updated for every i in U before the commit test; committed rows keep being
  processed by Core and Coda in later loops with input Emb(y_i); block positions that
  hold a given (non-mask) id are never in U and carry h~ like unresolved ones.

Precision: ``precision="fp64"`` computes everything in float64 from the given weights.
``precision="bf16"`` takes the decisions in the CUDA kernels' precision: every matrix
weight and every operand of a matrix product (normed activations, q/k/v, attention
probabilities, attention output, SwiGLU output, the readout state fed to the LM head)
is rounded to bfloat16 (nearest, ties to even) at the point where the kernels round it;
accumulation stays float64.  ``dtype=np.float32`` trades accuracy for speed at the
Qwen3 shapes.

Pins (tests/test_oracle_pins.py, CPU): brute-force primitives, entropy and sigmoid closed
forms, the commit-disabled step against an unrolled non-shared stack, K = 1 against a plain
masked-DLM step, the depth fallback against a position-by-position recursion, the layer and
KV-buffer counts the pages print, halting and rule traces built by hand, Eq. 3 on the loop
inputs, block decoding's step counts, append against one longer prefill, the sampler against
numpy's Philox generator and a chi-square test, and planted mistakes that each fail a pin.
The pages print no worked example with values, so absolute values on random weights are
parity unpinned beyond these structural pins.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional

import numpy as np

RULE_PAPER = 0
RULE_PER_TOKEN = 1


# ----------------------------------------------------------------------------------
# primitives
# ----------------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 value of x (via float32, ties to even), in x's float type.

    On the float32 bit pattern: add 0x7FFF plus the lowest kept bit, clear the 16 low bits
    (no finite pattern, nor infinity, overflows 32 bits doing so)."""
    x = np.asarray(x)
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32).astype(x.dtype)


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rope_cos_sin(positions: np.ndarray, head_dim: int, base: float, dtype) -> tuple:
    """Rotary angles pos * base^(-2j/hd), j = 0..hd/2-1 (computed in float64)."""
    j = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * j / head_dim)
    ang = positions.astype(np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang).astype(dtype), np.sin(ang).astype(dtype)


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE. x: [T, heads, hd]; cos/sin: [T, hd/2]."""
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, visible: np.ndarray,
              bf16: bool) -> np.ndarray:
    """softmax(q k^T / sqrt(hd)) v per query head; query head h reads KV head h // (nq/nkv).

    q: [Tq, nq, hd]; k, v: [Tk, nkv, hd]; visible: [Tq, Tk] bool.
    With bf16, the probabilities enter the value product rounded to bfloat16 while the
    normaliser is the sum of the unrounded ones (the kernels' precision).
    """
    Tq, nq, hd = q.shape
    nkv = k.shape[1]
    group = nq // nkv
    out = np.zeros((Tq, nq, hd), dtype=q.dtype)
    scale = 1.0 / math.sqrt(hd)
    for h in range(nq):
        kh = h // group
        s = (q[:, h, :] @ k[:, kh, :].T) * scale
        s = np.where(visible, s, -np.inf)
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        denom = p.sum(axis=-1, keepdims=True)
        pv = round_bf16(p) if bf16 else p
        out[:, h, :] = (pv @ v[:, kh, :]) / denom
    return out


# ----------------------------------------------------------------------------------
# decisions of one loop ([digest] "Method steps" (3)-(5))
# ----------------------------------------------------------------------------------

def commit_set(H: np.ndarray, a: np.ndarray, s: int, K: int, rule: int, tau: float, lam: float) -> np.ndarray:
    """Commit mask over the unresolved positions of loop s.

    PAPER: H <= tau (step (3)).  PER_TOKEN: H <= tau, or a >= lam, or the last loop."""
    if rule == RULE_PAPER:
        return H <= tau
    return (H <= tau) | (a >= lam) | (s == K)


def halting_mean(a: np.ndarray, unresolved: np.ndarray) -> float:
    """Step (4): the mean cumulative halt of the positions still unresolved after this loop's
    commits.  The pages say "the unresolved positions" without fixing when; the reading taken
    here is U once B^(s) has left it: positions committed in this or an earlier loop, and
    given ids, do not count.  0 when U is empty."""
    return float(np.mean(a[unresolved])) if unresolved.any() else 0.0


def halts(n_left: int, mean_a_left: float, s: int, K: int, rule: int, lam: float) -> bool:
    """Step (4): the loop ends when nothing is unresolved, at s = K, or (PAPER) when the mean
    cumulative halt of the unresolved positions reaches the threshold."""
    if n_left == 0 or s == K:
        return True
    return rule == RULE_PAPER and mean_a_left >= lam


# ----------------------------------------------------------------------------------
# sampling the committed token (digest "Method steps", Algorithm 1 (3): each committed
# position samples y_i ~ p_i^(s)); counter-based random numbers so that any other
# implementation can draw the same ones
# ----------------------------------------------------------------------------------

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
_LO32 = np.uint64(0xFFFFFFFF)
_PHILOX_M = (np.uint64(0xD2E7470EE14C6C93), np.uint64(0xCA5A826395121157))
_PHILOX_W = (np.uint64(0x9E3779B97F4A7C15), np.uint64(0xBB67AE8584CAA73B))


def _mulhilo64(a: np.ndarray, b: np.uint64):
    """(high, low) 64-bit halves of the 128-bit products a * b, through 32-bit limbs."""
    s32 = np.uint64(32)
    a0, a1 = a & _LO32, a >> s32
    b0, b1 = b & _LO32, b >> s32
    p00, p01, p10, p11 = a0 * b0, a0 * b1, a1 * b0, a1 * b1
    mid = (p00 >> s32) + (p01 & _LO32) + (p10 & _LO32)
    hi = p11 + (p01 >> s32) + (p10 >> s32) + (mid >> s32)
    return hi, a * b


def philox4x64(counter: np.ndarray, key) -> np.ndarray:
    """Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1,
    2, 3", SC 2011): ten rounds of two 64 x 64 -> 128-bit multiplications and xors, the key
    bumped by the Weyl constants between rounds.  counter [..., 4] uint64, key (2,) -> [..., 4]."""
    with np.errstate(over="ignore"):
        x = [np.asarray(counter, dtype=np.uint64)[..., i].copy() for i in range(4)]
        k0, k1 = np.uint64(key[0]), np.uint64(key[1])
        for r in range(10):
            if r:
                k0, k1 = k0 + _PHILOX_W[0], k1 + _PHILOX_W[1]
            hi0, lo0 = _mulhilo64(x[0], _PHILOX_M[0])
            hi1, lo1 = _mulhilo64(x[2], _PHILOX_M[1])
            x = [hi1 ^ x[1] ^ k0, lo1, hi0 ^ x[3] ^ k1, lo0]
    return np.stack(x, axis=-1)


def gumbel_scores(z: np.ndarray, key, position: int, loop: int) -> np.ndarray:
    """z_v + g_v with g_v = -log(-log(u_v)), u_v uniform in (0, 1) from the 53 high bits of
    Philox4x64-10 output (v mod 4) at counter (v div 4, position, loop, 0) under ``key``."""
    V = z.shape[0]
    nb = (V + 3) // 4
    ctr = np.zeros((nb, 4), dtype=np.uint64)
    ctr[:, 0] = np.arange(nb, dtype=np.uint64)
    ctr[:, 1] = np.uint64(position)
    ctr[:, 2] = np.uint64(loop)
    bits = philox4x64(ctr, key).reshape(-1)[:V]
    u = ((bits >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53
    g = -np.log(-np.log(u))
    return z.astype(np.float64) + g


def gumbel_argmax(z: np.ndarray, key, position: int, loop: int) -> int:
    """A draw from softmax(z) by the Gumbel-max construction (lowest index on ties)."""
    return int(np.argmax(gumbel_scores(z, key, position, loop)))


def forced_pick(H_by_pos: Dict[int, float]) -> int:
    """Step (5): the lowest-entropy unresolved position (lowest index on ties)."""
    return min(H_by_pos.items(), key=lambda kv: (kv[1], kv[0]))[0]


def replay_decisions(block_ids: np.ndarray, mask_id: int, entropy: np.ndarray, cum_halt: np.ndarray,
                     token_at, tau: float, lam: float, K: int, rule: int, mean_band: float = 1e-5) -> dict:
    """Re-take every decision of a step from given per-loop traces (entropy and cumulative
    halt [B,K,N], NaN outside U) with the rules above, in float32 like the traces.
    token_at(b, s, i) gives the token a position committing at loop s takes.  Returns
    tokens, exit_depth, loops_run and the near-threshold halting decisions it could not fix."""
    B, N = block_ids.shape
    tau32, lam32 = np.float32(tau), np.float32(lam)
    tokens = block_ids.astype(np.int64).copy()
    exit_depth = np.zeros((B, N), np.int64)
    loops = np.zeros(B, np.int64)
    ambiguous = []
    for b in range(B):
        U = block_ids[b] == mask_id
        n_commit = 0
        s_last = 1
        for s in range(1, K + 1):
            s_last = s
            idx = np.nonzero(U)[0]
            H = entropy[b, s - 1, idx].astype(np.float32)
            a = cum_halt[b, s - 1, idx].astype(np.float32)
            c = commit_set(H, a, s, K, rule, tau32, lam32)
            for i in idx[c]:
                tokens[b, i] = token_at(b, s, int(i))
                exit_depth[b, i] = s
            U[idx[c]] = False
            n_commit += int(c.sum())
            left = np.nonzero(U)[0]
            mean_a = halting_mean(cum_halt[b, s - 1].astype(np.float64), U)
            if len(left) and rule == RULE_PAPER and abs(mean_a - float(lam32)) < mean_band:
                ambiguous.append((b, s))
            if halts(len(left), np.float32(mean_a), s, K, rule, lam32):
                break
        if rule == RULE_PAPER and n_commit == 0 and U.any():
            i = forced_pick({int(i): float(entropy[b, s_last - 1, i]) for i in np.nonzero(U)[0]})
            tokens[b, i] = token_at(b, s_last, i)
            exit_depth[b, i] = s_last
        loops[b] = s_last
    return dict(tokens=tokens, exit_depth=exit_depth, loops_run=loops, ambiguous=ambiguous)


# ----------------------------------------------------------------------------------
# the model
# ----------------------------------------------------------------------------------

class Oracle:
    """ALoDLM inference, one sequence at a time, in plain NumPy.

    cfg: dict with hidden, n_q_heads, n_kv_heads, head_dim, inter, vocab, n_prelude,
    n_core, n_coda, k_max, rope_base, rms_eps, qk_norm, mask_id.
    weights: {"embed" [V,H], "lm_head" [V,H], "final_norm" [H], "exit_w" [H],
    "exit_b" float, "layers": list (model order) of {"attn_norm", "q", "k", "v", "o",
    "q_norm", "k_norm", "mlp_norm", "gate", "up", "down"}} as float arrays
    (row-major [out, in]).
    """

    def __init__(self, cfg: dict, weights: dict, precision: str = "fp64", dtype=np.float64):
        assert precision in ("fp64", "bf16")
        self.cfg = dict(cfg)
        self.W = weights
        self.bf16 = precision == "bf16"
        self.dt = dtype
        self.layer_execs = 0          # layer applications in the last denoise_step (per sequence, summed)
        self._layer_cache: Dict[int, dict] = {}
        n_params = sum(int(np.prod(np.shape(v))) for lw in self._layer_list() for v in lw.values())
        self._cache_layers = n_params < 200_000_000
        self.kv = None

    # --- weights ------------------------------------------------------------------

    def _layer_list(self):
        L = self.W["layers"]
        return L if isinstance(L, list) else [L[i] for i in sorted(L)]

    def _mat(self, a):
        if self.bf16:  # the rounding is done on float32 either way
            return round_bf16(np.asarray(a, dtype=np.float32)).astype(self.dt, copy=False)
        return np.asarray(a, dtype=self.dt)

    def _vec(self, a):
        # norm gains and the ExitGate weight are float32 in the kernels: no bf16 rounding
        return np.asarray(np.asarray(a, dtype=np.float32), dtype=self.dt)

    def layer_weights(self, idx: int) -> dict:
        if idx in self._layer_cache:
            return self._layer_cache[idx]
        src = self.W["layers"][idx]
        lw = {k: (self._vec(v) if np.ndim(v) == 1 else self._mat(v)) for k, v in src.items()}
        if self._cache_layers:
            self._layer_cache[idx] = lw
        return lw

    def _global(self, key):
        if ("g", key) not in self._layer_cache:
            v = self.W[key]
            self._layer_cache[("g", key)] = self._vec(v) if np.ndim(v) == 1 else self._mat(v)
        return self._layer_cache[("g", key)]

    def _act(self, x):
        return round_bf16(x) if self.bf16 else x

    # --- slots of the depth-aware KV cache ---------------------------------------------
    # [digest] "Technical novelty" and "Prerequisites": a shared Core layer produces a
    # different KV at every loop depth, so the cache keeps one buffer per (Core layer,
    # depth) beside one per Prelude and per Coda layer.

    def n_kv_slots(self, k_max: Optional[int] = None) -> int:
        c = self.cfg
        K = c["k_max"] if k_max is None else k_max
        return c["n_prelude"] + K * c["n_core"] + c["n_coda"]

    def core_layer_index(self, j: int) -> int:
        return self.cfg["n_prelude"] + j

    def coda_layer_index(self, j: int) -> int:
        return self.cfg["n_prelude"] + self.cfg["n_core"] + j

    # --- one decoder layer -------------------------------------------------------------

    def qkv(self, lw: dict, h: np.ndarray, positions: np.ndarray):
        """Normed input -> (q, k, v) after the per-head norms and RoPE."""
        c = self.cfg
        nq, nkv, hd = c["n_q_heads"], c["n_kv_heads"], c["head_dim"]
        x = self._act(rmsnorm(h, lw["attn_norm"], c["rms_eps"]))
        q = (x @ lw["q"].T).reshape(-1, nq, hd)
        k = (x @ lw["k"].T).reshape(-1, nkv, hd)
        v = (x @ lw["v"].T).reshape(-1, nkv, hd)
        if c["qk_norm"]:
            q = rmsnorm(q, lw["q_norm"], c["rms_eps"])
            k = rmsnorm(k, lw["k_norm"], c["rms_eps"])
        cos, sin = rope_cos_sin(positions, hd, c["rope_base"], self.dt)
        q = apply_rope(q, cos, sin)
        k = apply_rope(k, cos, sin)
        return self._act(q), self._act(k), self._act(v)

    def finish_layer(self, lw: dict, h: np.ndarray, q, k_all, v_all, visible) -> np.ndarray:
        """Attention over (k_all, v_all), output projection, residual, SwiGLU MLP, residual."""
        c = self.cfg
        o = attention(q, k_all, v_all, visible, self.bf16)
        o = self._act(o.reshape(o.shape[0], -1))
        h = h + o @ lw["o"].T
        x = self._act(rmsnorm(h, lw["mlp_norm"], c["rms_eps"]))
        a = self._act(silu(x @ lw["gate"].T) * (x @ lw["up"].T))
        return h + a @ lw["down"].T

    # --- prefill: the depth-aware KV cache ---------------------------------------------

    def prefill(self, prefix_ids: np.ndarray, exit_depth: Optional[np.ndarray] = None) -> dict:
        """Build the depth-aware KV cache of the prefix.

        [digest] "Technical novelty"/"Prerequisites": each prefix position is served at the
        matching loop depth, falling back to the deepest depth it reached.  Position j with
        exit depth e_j runs the Core e_j times; for depth d > e_j its Core KV is its depth-e_j
        KV.  Keys at Core depth d are therefore read at depth min(d, e_k).  The Coda runs
        once, on each position's depth-e_j state.  Attention is causal over the prefix.

        Stores self.kv[b][("prelude", l) | ("core", c, d) | ("coda", j)] = (K, V), each
        [P, nkv, hd]; returns it.
        """
        c = self.cfg
        K = c["k_max"]
        prefix_ids = np.asarray(prefix_ids)
        B, P = prefix_ids.shape
        if exit_depth is None:
            exit_depth = np.full((B, P), K, dtype=np.int64)
        exit_depth = np.asarray(exit_depth)
        assert exit_depth.min() >= 1 and exit_depth.max() <= K
        emb = self._global("embed")
        pos = np.arange(P)
        causal = pos[None, :] <= pos[:, None]
        self.kv = []
        for b in range(B):
            kv = {}
            h = emb[prefix_ids[b]].astype(self.dt)
            for l in range(c["n_prelude"]):
                lw = self.layer_weights(l)
                q, k, v = self.qkv(lw, h, pos)
                kv[("prelude", l)] = (k, v)
                h = self.finish_layer(lw, h, q, k, v, causal)
            e = exit_depth[b]
            h_exit = h.copy()
            for d in range(1, K + 1):
                act = np.nonzero(e >= d)[0]
                for j in range(c["n_core"]):
                    lw = self.layer_weights(self.core_layer_index(j))
                    if d == 1:
                        k_d = np.zeros((P, c["n_kv_heads"], c["head_dim"]), dtype=self.dt)
                        v_d = np.zeros_like(k_d)
                    else:
                        # positions that stopped before depth d keep their deepest KV
                        k_d, v_d = (x.copy() for x in kv[("core", j, d - 1)])
                    kv[("core", j, d)] = (k_d, v_d)
                    if len(act) == 0:
                        continue
                    q, k, v = self.qkv(lw, h[act], pos[act])
                    k_d[act], v_d[act] = k, v
                    h[act] = self.finish_layer(lw, h[act], q, k_d, v_d, causal[act])
                h_exit[e == d] = h[e == d]
            h = h_exit
            for j in range(c["n_coda"]):
                lw = self.layer_weights(self.coda_layer_index(j))
                q, k, v = self.qkv(lw, h, pos)
                kv[("coda", j)] = (k, v)
                h = self.finish_layer(lw, h, q, k, v, causal)
            self.kv.append(kv)
        self.prefix_len = P
        return self.kv

    def append(self, ids: np.ndarray, exit_depth: Optional[np.ndarray] = None) -> dict:
        """Extend the cached prefix by N positions P..P+N-1 holding ``ids`` (a decoded block).

        [digest] "Method steps", Algorithm 1 (5): the committed tokens are written into the
        sequence, which later blocks attend to as context; "Technical novelty": every
        position is served at its own loop depth, the deepest it reached standing in for
        deeper ones.  The new positions go through exactly what ``prefill`` does for prefix
        positions -- Prelude, the Core e_j times (Core KV at depth d > e_j = the depth-e_j KV),
        the Coda once on the depth-e_j state -- attending to every cached position (at its
        own slot, fallback already resolved) and causally to each other.  ``exit_depth``
        [B, N] in 1..k_max (default k_max).  Extends self.kv in place; returns it.
        """
        c = self.cfg
        K = c["k_max"]
        assert self.kv is not None, "prefill first"
        ids = np.asarray(ids)
        B, N = ids.shape
        P = self.prefix_len
        if exit_depth is None:
            exit_depth = np.full((B, N), K, dtype=np.int64)
        exit_depth = np.asarray(exit_depth)
        assert exit_depth.min() >= 1 and exit_depth.max() <= K
        emb = self._global("embed")
        pos = P + np.arange(N)
        # new row i sees every cached position and the new positions up to itself
        vis = np.concatenate([np.ones((N, P), dtype=bool), np.tril(np.ones((N, N), dtype=bool))], axis=1)

        def extend(key, k_new, v_new):
            kp, vp = kv[key]
            kv[key] = (np.concatenate([kp, k_new], axis=0), np.concatenate([vp, v_new], axis=0))
            return kv[key]

        for b in range(B):
            kv = self.kv[b]
            h = emb[ids[b]].astype(self.dt)
            for l in range(c["n_prelude"]):
                lw = self.layer_weights(l)
                q, k, v = self.qkv(lw, h, pos)
                k_all, v_all = extend(("prelude", l), k, v)
                h = self.finish_layer(lw, h, q, k_all, v_all, vis)
            e = exit_depth[b]
            h_exit = h.copy()
            for d in range(1, K + 1):
                act = np.nonzero(e >= d)[0]
                for j in range(c["n_core"]):
                    lw = self.layer_weights(self.core_layer_index(j))
                    if d == 1:
                        k_new = np.zeros((N, c["n_kv_heads"], c["head_dim"]), dtype=self.dt)
                        v_new = np.zeros_like(k_new)
                    else:
                        # new positions that stopped before depth d keep their deepest KV
                        k_new, v_new = (x[P:].copy() for x in kv[("core", j, d - 1)])
                    if len(act):
                        q, k, v = self.qkv(lw, h[act], pos[act])
                        k_new[act], v_new[act] = k, v
                    k_all, v_all = extend(("core", j, d), k_new, v_new)
                    if len(act):
                        h[act] = self.finish_layer(lw, h[act], q, k_all, v_all, vis[act])
                h_exit[e == d] = h[e == d]
            h = h_exit
            for j in range(c["n_coda"]):
                lw = self.layer_weights(self.coda_layer_index(j))
                q, k, v = self.qkv(lw, h, pos)
                k_all, v_all = extend(("coda", j), k, v)
                h = self.finish_layer(lw, h, q, k_all, v_all, vis)
        self.prefix_len = P + N
        return self.kv

    # --- one layer over the block against the cached prefix ----------------------------

    def block_layer(self, b: int, key, lw: dict, h: np.ndarray) -> np.ndarray:
        """The block attends to every cached prefix position (slot ``key``) and to itself."""
        P = self.prefix_len
        N = h.shape[0]
        pos = P + np.arange(N)
        q, k, v = self.qkv(lw, h, pos)
        kp, vp = self.kv[b][key]
        k_all = np.concatenate([kp, k], axis=0)
        v_all = np.concatenate([vp, v], axis=0)
        visible = np.ones((N, P + N), dtype=bool)
        self.layer_execs += 1
        return self.finish_layer(lw, h, q, k_all, v_all, visible)

    def readout(self, r: np.ndarray):
        """LMHead and ExitGate on readout states r [n, H].

        [digest] "Core method": p_i = softmax(LMHead(r_i)); entropy H_i = -sum p log p (nats);
        lambda_i = sigmoid(ExitGate(r_i)).  Returns (H, y = argmax, lam, z = logits).
        """
        W = self._global("lm_head")
        z = self._act(r) @ W.T
        m = z.max(axis=-1, keepdims=True)
        logZ = m + np.log(np.exp(z - m).sum(axis=-1, keepdims=True))
        logp = z - logZ
        p = np.exp(logp)
        H = -(p * logp).sum(axis=-1)
        y = np.argmax(z, axis=-1)
        g = r @ self._global("exit_w") + float(self.W["exit_b"])
        return H, y, sigmoid(g), z

    def merge(self, committed: np.ndarray, tok: np.ndarray, h_tilde: np.ndarray) -> np.ndarray:
        """[digest] Eq. 3: h_i^(s) = Emb(y_i) for a committed position, h~_i^(s) otherwise."""
        emb = self._global("embed")
        return np.where(committed[:, None], emb[tok], h_tilde)

    # --- the denoising step --------------------------------------------------------------

    def denoise_step(self, block_ids: np.ndarray, tau: float, lam: float, k_max: int,
                     rule: int = RULE_PAPER, follow: Optional[dict] = None, band=1e-3,
                     logit_rows: Optional[List[tuple]] = None, sample_key=None) -> dict:
        """One denoising step, [digest] "Method steps" Algorithm 1 (1)-(5) and Eq. 3.

        block_ids [B, N]; positions holding mask_id form U.  ``lam`` is the halting
        threshold (q in the pages).  ``follow`` (optional) holds another run's decisions
        {"tokens" [B,N], "exit_depth" [B,N], "loops_run" [B]}: at a decision whose deciding
        value lies within the band of its threshold, the oracle takes that run's decision and
        records it in "followed" (with its own decision and the margin).  ``band`` is one
        number for every kind of decision, or a dict with keys "entropy" (a commit on H <= tau,
        and the forced pick when the two lowest entropies are that close), "halt" (a decision
        on a cumulative halt or its mean) and "argmax" (the top-two score gap; the other run's
        token is taken only if its score lies within the band of the maximum); each value is
        a number or a sequence indexed by loop s - 1 (its last entry for deeper loops).
        band=inf follows every decision.  ``logit_rows``: (b, s, i) triples whose logits are returned.
        ``sample_key`` (two integers): committed tokens are drawn from p_i^(s) by Gumbel-max
        (``gumbel_argmax`` at position b * N + i, loop s) instead of taken greedily.

        Returns tokens, exit_depth, entropy/halt/cum_halt [B,K,N] (NaN where not computed),
        loops_run [B], active_rows [K], readout_rows [K]; per sequence b, lists of
        [loops, N, H] arrays: r (readout states r^(s)), h_in (loop inputs h^(s-1)) and
        h_tilde (Core outputs); logits {(b,s,i): z}, followed, committed_per_step [B].
        """
        c = self.cfg
        assert self.kv is not None, "prefill first"
        assert 1 <= k_max <= c["k_max"]
        block_ids = np.asarray(block_ids)
        B, N = block_ids.shape
        K = k_max
        mask_id = c["mask_id"]
        emb = self._global("embed")
        nan = np.full((B, K, N), np.nan)
        out = dict(tokens=block_ids.astype(np.int64).copy(), exit_depth=np.zeros((B, N), np.int64),
                   entropy=nan.copy(), halt=nan.copy(), cum_halt=nan.copy(),
                   loops_run=np.zeros(B, np.int64), active_rows=np.zeros(K, np.int64),
                   readout_rows=np.zeros(K, np.int64), r=[], h_in=[], h_tilde=[], logits={}, followed=[],
                   committed_per_step=np.zeros(B, np.int64))
        want_logits = set(logit_rows or [])
        self.layer_execs = 0

        bands = band if isinstance(band, dict) else dict(entropy=band, halt=band, argmax=band)

        def band_at(kind, s):
            v = bands[kind]
            return float(v) if np.ndim(v) == 0 else float(v[min(s, len(v)) - 1])

        def near(x, thr, width):
            return follow is not None and abs(float(x) - float(thr)) < width

        for b in range(B):
            # (1) U = masked positions; h^(0) = Prelude(x); a = 0; C = empty
            U = block_ids[b] == mask_id
            tok = block_ids[b].astype(np.int64).copy()
            committed = np.zeros(N, dtype=bool)
            a = np.zeros(N, dtype=self.dt)
            h = emb[block_ids[b]].astype(self.dt)
            for l in range(c["n_prelude"]):
                h = self.block_layer(b, ("prelude", l), self.layer_weights(l), h)
            rs, h_ins, h_tildes = [], [], []
            n_committed = 0
            last_H = None
            s_last = 0
            for s in range(1, K + 1):
                s_last = s
                out["active_rows"][s - 1] += N
                # (2) h~ = Core(h^(s-1)) against prefix Core KV at depth s; r = Coda(h~)
                h_ins.append(h)
                ht = h
                for j in range(c["n_core"]):
                    ht = self.block_layer(b, ("core", j, s), self.layer_weights(self.core_layer_index(j)), ht)
                h_tildes.append(ht)
                hc = ht
                for j in range(c["n_coda"]):
                    hc = self.block_layer(b, ("coda", j), self.layer_weights(self.coda_layer_index(j)), hc)
                r = rmsnorm(hc, self._global("final_norm"), c["rms_eps"])
                rs.append(r)
                idx = np.nonzero(U)[0]
                out["readout_rows"][s - 1] += len(idx)
                H, y, lmb, z = self.readout(r[idx])
                for t, i in enumerate(idx):
                    if (b, s, int(i)) in want_logits:
                        out["logits"][(b, s, int(i))] = z[t]
                # (4) cumulative halting a <- a + (1 - a) lambda, for every i in U
                a[idx] = a[idx] + (1.0 - a[idx]) * lmb
                out["entropy"][b, s - 1, idx] = H
                out["halt"][b, s - 1, idx] = lmb
                out["cum_halt"][b, s - 1, idx] = a[idx]
                last_H = dict(zip(idx.tolist(), H.tolist()))
                # greedy token choice (lowest id on ties), or a Gumbel-max draw
                y = y.astype(np.int64).copy()
                scores = z
                if sample_key is not None:
                    scores = np.stack([gumbel_scores(z[t], sample_key, b * N + int(idx[t]), s)
                                       for t in range(len(idx))]) if len(idx) else z
                    y = np.argmax(scores, axis=-1).astype(np.int64) if len(idx) else y
                band_h, band_a, band_z = band_at("entropy", s), band_at("halt", s), band_at("argmax", s)
                if follow is not None:
                    for t in range(len(idx)):
                        top2 = np.partition(scores[t], -2)[-2:]
                        i = int(idx[t])
                        other = int(follow["tokens"][b, i])
                        if (top2[1] - top2[0] < band_z and follow["exit_depth"][b, i] == s
                                and 0 <= other < scores.shape[1] and scores[t][other] >= top2[1] - band_z):
                            out["followed"].append(dict(b=b, s=s, i=i, kind="argmax",
                                                        margin=float(top2[1] - top2[0]), own=int(y[t]),
                                                        taken=other))
                            y[t] = other
                # (3) commit set B^(s)
                commit = commit_set(H, a[idx], s, K, rule, tau, lam)
                for t, i in enumerate(idx):
                    dec = bool(commit[t])
                    if rule == RULE_PAPER:
                        is_near = near(H[t], tau, band_h)
                        margin = H[t] - tau
                    else:
                        is_near = s < K and (near(H[t], tau, band_h) or near(a[i], lam, band_a))
                        margin = min(abs(H[t] - tau), abs(a[i] - lam))
                    if is_near:
                        gpu = bool(follow["exit_depth"][b, i] == s)
                        out["followed"].append(dict(b=b, s=s, i=int(i), kind="commit",
                                                    margin=float(margin), own=bool(dec), taken=gpu))
                        dec = gpu
                    commit[t] = dec
                ci = idx[commit]
                tok[ci] = y[commit]
                out["exit_depth"][b, ci] = s
                U[ci] = False
                committed[ci] = True
                n_committed += len(ci)
                h = self.merge(committed, tok, ht)
                # (4) halting
                mean_a = halting_mean(a, U)
                stop = halts(int(U.sum()), mean_a, s, K, rule, lam)
                if rule == RULE_PAPER and U.any() and s < K and near(mean_a, lam, band_a):
                    gpu = bool(follow["loops_run"][b] == s)
                    out["followed"].append(dict(b=b, s=s, i=-1, kind="halt",
                                                margin=float(mean_a - lam), own=stop, taken=gpu))
                    stop = gpu
                if stop:
                    break
            # (5) forced progress: nothing committed in this step -> lowest entropy of the last loop
            if rule == RULE_PAPER and n_committed == 0 and U.any():
                band_h, band_z = band_at("entropy", s_last), band_at("argmax", s_last)
                cand = sorted(last_H.items(), key=lambda kv: (kv[1], kv[0]))
                i_star = forced_pick(last_H)
                if follow is not None and len(cand) > 1 and cand[1][1] - cand[0][1] < band_h:
                    gpu_i = [i for i in last_H if follow["exit_depth"][b, i] == s_last
                             and last_H[i] <= cand[0][1] + band_h]
                    if gpu_i:
                        out["followed"].append(dict(b=b, s=s_last, i=int(i_star), kind="forced",
                                                    margin=float(cand[1][1] - cand[0][1]), own=int(i_star),
                                                    taken=int(gpu_i[0])))
                        i_star = gpu_i[0]
                z_star = self.readout(rs[-1][[i_star]])[3][0]
                if sample_key is not None:
                    z_star = gumbel_scores(z_star, sample_key, b * N + int(i_star), s_last)
                y_star = int(np.argmax(z_star))
                if follow is not None and follow["exit_depth"][b, i_star] == s_last:
                    top2 = np.partition(z_star, -2)[-2:]
                    other = int(follow["tokens"][b, i_star])
                    if top2[1] - top2[0] < band_z and 0 <= other < z_star.shape[0] and \
                            z_star[other] >= top2[1] - band_z:
                        out["followed"].append(dict(b=b, s=s_last, i=int(i_star), kind="argmax",
                                                    margin=float(top2[1] - top2[0]), own=y_star, taken=other))
                        y_star = other
                tok[i_star] = y_star
                out["exit_depth"][b, i_star] = s_last
                U[i_star] = False
                n_committed = 1
            out["tokens"][b] = tok
            out["loops_run"][b] = s_last
            out["committed_per_step"][b] = n_committed
            out["r"].append(np.stack(rs))
            out["h_in"].append(np.stack(h_ins))
            out["h_tilde"].append(np.stack(h_tildes))
        return out


def decode_block(oracle: Oracle, block_ids: np.ndarray, tau: float, lam: float, k_max: int,
                 rule: int = RULE_PAPER, max_steps: int = 0, follow_steps: Optional[List[dict]] = None,
                 band=1e-3, sample_seed: Optional[int] = None) -> dict:
    """Denoising steps over one block until no [MASK] is left, [digest] "Method steps",
    Algorithm 1 (5): after each step the committed tokens are written into the sequence and
    the next denoising step starts, until no [MASK] remains.

    Every step sees the same prefix KV (the block is re-embedded from its ids each step); step
    t + 1 takes the tokens of step t as its block ids.  The whole batch steps together; a
    sequence without masks still runs a step (its U is empty, so nothing changes), and stops
    counting steps once its block is complete.  ``max_steps`` (0 = N) bounds the steps.
    ``follow_steps``: per step, another run's decisions (the ``follow`` argument of
    ``Oracle.denoise_step``).  ``sample_seed``: draw the committed tokens (key (seed, step)).

    Returns tokens [B,N] (final), commit_step [B,N] (1-based step that committed the
    position; 0 for given ids and positions never committed), commit_depth [B,N] (the loop s
    of that step), steps_run [B] (steps that had masks at their start), loops [steps, B]
    (loops run per step), steps (steps taken), and the per-step outputs ("per_step").
    """
    mask_id = oracle.cfg["mask_id"]
    ids = np.asarray(block_ids).astype(np.int64).copy()
    B, N = ids.shape
    limit = max_steps if max_steps > 0 else N
    commit_step = np.zeros((B, N), np.int64)
    commit_depth = np.zeros((B, N), np.int64)
    steps_run = np.zeros(B, np.int64)
    loops, per_step = [], []
    t = 0
    while t < limit and (ids == mask_id).any():
        t += 1
        had_masks = (ids == mask_id).any(axis=1)
        follow = follow_steps[t - 1] if follow_steps is not None and t - 1 < len(follow_steps) else None
        key = None if sample_seed is None else (int(sample_seed), t)
        out = oracle.denoise_step(ids, tau, lam, k_max, rule, follow=follow, band=band, sample_key=key)
        new = out["exit_depth"] > 0
        commit_step[new] = t
        commit_depth[new] = out["exit_depth"][new]
        steps_run[had_masks] = t
        loops.append(out["loops_run"].copy())
        per_step.append(out)
        ids = out["tokens"].astype(np.int64).copy()
    return dict(tokens=ids, commit_step=commit_step, commit_depth=commit_depth, steps_run=steps_run,
                loops=np.array(loops, dtype=np.int64).reshape(t, B), steps=t, per_step=per_step)
