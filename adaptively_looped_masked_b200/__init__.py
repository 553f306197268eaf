"""Python binding of libalodlm.so (the ALoDLM denoising-step library, sm_100a).

Argument marshalling only: tensors are passed to the C ABI as raw device pointers and
every step of the computation runs in the library's CUDA kernels.  There is no fallback:
if the shared object is missing or cannot be loaded, importing the binding's entry points
raises.  PyTorch is used for device memory and streams.

Names follow the C ABI (include/alodlm.h): ``Handle.create``, ``prefill``, ``denoise_step``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .build import LIB_PATH, build as build_library  # noqa: F401

RULE_PAPER = 0
RULE_PER_TOKEN = 1
DTYPE_BF16 = 0
DTYPE_F32 = 1

STATUS = {0: "OK", -1: "EINVAL", -2: "ENOMEM", -3: "ECUDA", -4: "EDEVICE", -5: "ETIMEOUT", -6: "ESTATE"}
N_KCLASS = 9


class AlodlmError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("hidden", "n_q_heads", "n_kv_heads", "head_dim", "inter", "vocab",
                                            "n_prelude", "n_core", "n_coda", "k_max", "max_batch", "max_prefix",
                                            "max_block")] + [
        ("rope_base", ctypes.c_float), ("rms_eps", ctypes.c_float), ("mask_id", ctypes.c_int),
        ("qk_norm", ctypes.c_int), ("mem_limit_bytes", ctypes.c_size_t), ("debug_dump", ctypes.c_int)]


LAYER_FIELDS = ("attn_norm", "q", "k", "v", "o", "q_norm", "k_norm", "mlp_norm", "gate", "up", "down")


class LayerW(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in LAYER_FIELDS]


class Weights(ctypes.Structure):
    _fields_ = [("matrix_dtype", ctypes.c_int), ("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("final_norm", ctypes.c_void_p), ("exit_w", ctypes.c_void_p), ("exit_b", ctypes.c_float),
                ("layers", ctypes.POINTER(LayerW))]


class StepOut(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("tokens", "exit_depth", "entropy", "halt", "cum_halt", "loops_run",
                                               "active_rows", "readout_rows")]


class DecodeOut(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("tokens", "commit_step", "commit_depth", "steps_run", "loops", "rows")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it is not built: there is no other implementation)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libalodlm.so is not built ({LIB_PATH}); run adaptively_looped_masked_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci, cf, csz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.alodlm_create.argtypes = [ctypes.POINTER(Cfg), ctypes.POINTER(Weights), vp, ctypes.POINTER(vp)]
        L.alodlm_prefill.argtypes = [vp, vp, ci, ci, vp]
        L.alodlm_append.argtypes = [vp, vp, ci, ci, vp]
        L.alodlm_denoise_step.argtypes = [vp, vp, ci, ci, cf, cf, ci, ci, ctypes.POINTER(StepOut)]
        L.alodlm_decode_block.argtypes = [vp, vp, ci, ci, cf, cf, ci, ci, ci, ctypes.POINTER(DecodeOut),
                                          ctypes.POINTER(ci)]
        u64 = ctypes.c_uint64
        L.alodlm_denoise_step_sampled.argtypes = [vp, vp, ci, ci, cf, cf, ci, ci, u64, u64, ctypes.POINTER(StepOut)]
        L.alodlm_decode_block_sampled.argtypes = [vp, vp, ci, ci, cf, cf, ci, ci, ci, u64, ctypes.POINTER(DecodeOut),
                                                  ctypes.POINTER(ci)]
        L.alodlm_sync.argtypes = [vp]
        L.alodlm_inject_wait_timeout.argtypes = [vp]
        L.alodlm_destroy.argtypes = [vp]
        L.alodlm_destroy.restype = None
        L.alodlm_last_error.argtypes = [vp]
        L.alodlm_last_error.restype = ctypes.c_char_p
        L.alodlm_debug_state.argtypes = [vp, ci, ci, vp]
        L.alodlm_kv_slot.argtypes = [vp, ci, ci, ci, ci, vp]
        L.alodlm_step_stats.argtypes = [vp, ctypes.POINTER(ci), ctypes.POINTER(ctypes.c_double),
                                        ctypes.POINTER(ci), ctypes.POINTER(ctypes.c_double),
                                        ctypes.POINTER(ctypes.c_double)]
        L.alodlm_set_timing.argtypes = [vp, ci]
        L.alodlm_set_graphs.argtypes = [vp, ci]
        L.alodlm_kernel_class_name.argtypes = [ci]
        L.alodlm_kernel_class_name.restype = ctypes.c_char_p
        L.alodlm_gemm_bf16.argtypes = [vp, vp, vp, ci, ci, ci, vp, csz, vp]
        L.alodlm_gemm_bf16_noalloc.argtypes = [vp, vp, vp, ci, ci, ci, vp, vp]
        i32p = ctypes.POINTER(ctypes.c_int32)
        L.alodlm_plan_gemm.argtypes = [ci, ci, ci, i32p]
        L.alodlm_plan_gemm_noalloc.argtypes = [ci, ci, ci, ci, i32p]
        L.alodlm_plan_attention.argtypes = [ci, ci, ci, ci, ci, ci, ci, ci, i32p]
        for f in ("alodlm_create", "alodlm_prefill", "alodlm_append", "alodlm_denoise_step",
                  "alodlm_denoise_step_sampled", "alodlm_decode_block_sampled", "alodlm_decode_block", "alodlm_sync", "alodlm_debug_state",
                  "alodlm_kv_slot", "alodlm_step_stats", "alodlm_set_timing", "alodlm_set_graphs",
                  "alodlm_gemm_bf16", "alodlm_gemm_bf16_noalloc", "alodlm_plan_gemm", "alodlm_plan_gemm_noalloc",
                  "alodlm_plan_attention"):
            getattr(L, f).restype = ci
        _lib = L
    return _lib


def _plan(fn: str, n_out: int, *args) -> tuple:
    out = (ctypes.c_int32 * n_out)()
    rc = getattr(lib(), fn)(*args, out)
    if rc != 0:
        raise AlodlmError(rc, lib().alodlm_last_error(None).decode())
    return tuple(out)


def plan_gemm(M: int, N: int, K: int) -> dict:
    """The per-tile linear-layer kernel's partition (alodlm_plan_gemm); no device work."""
    bn, splits, kps, k_tiles = _plan("alodlm_plan_gemm", 4, M, N, K)
    return dict(bn=bn, splits=splits, kps=kps, k_tiles=k_tiles)


def plan_gemm_noalloc(M: int, N: int, K: int, num_sms: int) -> dict:
    """The allocation-free GEMM's stream-K partition (alodlm_plan_gemm_noalloc); no device work."""
    bn, grid, upc, max_seg, n_tiles, k_tiles = _plan("alodlm_plan_gemm_noalloc", 6, M, N, K, num_sms)
    return dict(bn=bn, grid=grid, upc=upc, max_seg=max_seg, n_tiles=n_tiles, k_tiles=k_tiles)


def plan_attention(packed_rows: int, n_kv_heads: int, n_seq: int, kv_len: int, causal: bool, num_sms: int,
                   two_tile_ok: bool, cluster16_ok: bool) -> dict:
    """One attention launch's partition (alodlm_plan_attention); no device work."""
    qtiles, two_tile, splits, kps, last_to_end = _plan("alodlm_plan_attention", 5, packed_rows, n_kv_heads, n_seq,
                                                       kv_len, int(causal), num_sms, int(two_tile_ok),
                                                       int(cluster16_ok))
    return dict(qtiles=qtiles, two_tile=two_tile, splits=splits, keys_per_split=kps, last_to_end=last_to_end)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def gemm_bf16(A: torch.Tensor, W: torch.Tensor, out: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """C = A @ W^T through the library's tcgen05 GEMM (A [M,K], W [N,K] bf16 -> f32 [M,N])."""
    M, K = A.shape
    N = W.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=A.device)
    if workspace is None:
        workspace = torch.zeros(64, dtype=torch.float32, device=A.device)  # the status word
    rc = lib().alodlm_gemm_bf16(_ptr(A), _ptr(W), _ptr(out), M, N, K, _ptr(workspace),
                                workspace.numel() * 4, _stream_ptr(stream))
    if rc:
        raise AlodlmError(rc, "alodlm_gemm_bf16 failed")
    return out


def gemm_bf16_noalloc(A: torch.Tensor, W: torch.Tensor, out: torch.Tensor, status: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """C = A @ W^T through the allocation-free entry point (scratch compiled into the library).
    ``out`` must be given: this call allocates nothing.  ``status`` (optional, device int32
    [1]) receives the call's status word (non-zero: a bounded wait timed out, C invalid)."""
    M, K = A.shape
    N = W.shape[0]
    if status is not None and (status.dtype != torch.int32 or status.numel() < 1):
        raise ValueError("status must be a device int32 tensor")
    rc = lib().alodlm_gemm_bf16_noalloc(_ptr(A), _ptr(W), _ptr(out), M, N, K, _ptr(status), _stream_ptr(stream))
    if rc:
        raise AlodlmError(rc, lib().alodlm_last_error(None).decode())
    return out


class Handle:
    """One model instance on the current CUDA device (wraps alodlm_t*)."""

    def __init__(self, shape, weights: dict, k_max: int, max_batch: int, max_prefix: int, max_block: int,
                 stream: Optional[torch.cuda.Stream] = None, debug_dump: bool = False, mem_limit_bytes: int = 0):
        L = lib()
        self.shape = shape
        self.k_max = k_max
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        cfg = Cfg(hidden=shape.hidden, n_q_heads=shape.n_q_heads, n_kv_heads=shape.n_kv_heads,
                  head_dim=shape.head_dim, inter=shape.inter, vocab=shape.vocab, n_prelude=shape.n_prelude,
                  n_core=shape.n_core, n_coda=shape.n_coda, k_max=k_max, max_batch=max_batch,
                  max_prefix=max_prefix, max_block=max_block, rope_base=shape.rope_base, rms_eps=shape.rms_eps,
                  mask_id=shape.mask_id, qk_norm=shape.qk_norm, mem_limit_bytes=mem_limit_bytes,
                  debug_dump=int(debug_dump))
        mat_dtype = weights["embed"].dtype
        dt = DTYPE_BF16 if mat_dtype == torch.bfloat16 else DTYPE_F32
        layers = (LayerW * len(weights["layers"]))()
        keep = []
        for i, lw in enumerate(weights["layers"]):
            for f in LAYER_FIELDS:
                t = lw[f]
                if t.dim() == 2 and t.dtype != mat_dtype:
                    raise ValueError("all weight matrices must share one dtype")
                if t.dim() == 1 and t.dtype != torch.float32:
                    t = t.float()
                    keep.append(t)
                setattr(layers[i], f, _ptr(t))
        fn, ew = weights["final_norm"].float(), weights["exit_w"].float()
        keep += [fn, ew]
        w = Weights(matrix_dtype=dt, embed=_ptr(weights["embed"]), lm_head=_ptr(weights["lm_head"]),
                    final_norm=_ptr(fn), exit_w=_ptr(ew), exit_b=float(weights["exit_b"]), layers=layers)
        h = ctypes.c_void_p()
        rc = L.alodlm_create(ctypes.byref(cfg), ctypes.byref(w), _stream_ptr(self.stream), ctypes.byref(h))
        if rc:
            raise AlodlmError(rc, L.alodlm_last_error(None).decode())
        self._h = h
        self.B = None
        self.N = None

    def _order_in(self):
        """The handle's stream waits for work already queued on torch's current stream."""
        cur = torch.cuda.current_stream()
        if cur != self.stream:
            self.stream.wait_stream(cur)

    def _order_out(self):
        """torch's current stream waits for the handle's stream (results visible to later ops)."""
        cur = torch.cuda.current_stream()
        if cur != self.stream:
            cur.wait_stream(self.stream)

    def _check(self, rc: int, what: str):
        if rc:
            raise AlodlmError(rc, f"{what}: {lib().alodlm_last_error(self._h).decode()}")

    def close(self):
        if getattr(self, "_h", None):
            lib().alodlm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def prefill(self, prefix_ids: torch.Tensor, exit_depth: Optional[torch.Tensor] = None):
        B, P = prefix_ids.shape
        ids = prefix_ids.to(torch.int32).contiguous()
        e = None if exit_depth is None else exit_depth.to(torch.int32).contiguous()
        self._keep = (ids, e)
        self._order_in()
        self._check(lib().alodlm_prefill(self._h, _ptr(ids), B, P, _ptr(e)), "prefill")
        self._order_out()
        self.B, self.P = B, P

    def append(self, ids: torch.Tensor, exit_depth: Optional[torch.Tensor] = None):
        """Append positions P..P+N-1 holding ids [B, N] to the cached prefix (alodlm_append);
        exit_depth [B, N] in 1..k_max or None (k_max)."""
        B, N = ids.shape
        ids = ids.to(torch.int32).contiguous()
        e = None if exit_depth is None else exit_depth.to(torch.int32).contiguous()
        self._keep_append = (ids, e)
        self._order_in()
        self._check(lib().alodlm_append(self._h, _ptr(ids), B, N, _ptr(e)), "append")
        self._order_out()
        self.P += N

    def alloc_outputs(self, B: int, N: int, k_max: int, device=None) -> dict:
        dev = device or torch.device("cuda", torch.cuda.current_device())
        i32, f32 = torch.int32, torch.float32
        return dict(tokens=torch.empty((B, N), dtype=i32, device=dev),
                    exit_depth=torch.empty((B, N), dtype=i32, device=dev),
                    entropy=torch.empty((B, k_max, N), dtype=f32, device=dev),
                    halt=torch.empty((B, k_max, N), dtype=f32, device=dev),
                    cum_halt=torch.empty((B, k_max, N), dtype=f32, device=dev),
                    loops_run=torch.empty((B,), dtype=i32, device=dev),
                    active_rows=torch.empty((k_max,), dtype=i32, device=dev),
                    readout_rows=torch.empty((k_max,), dtype=i32, device=dev))

    def denoise_step(self, block_ids: torch.Tensor, tau_H: float, lam: float, k_max: int,
                     rule: int = RULE_PAPER, out: Optional[dict] = None, sample: Optional[tuple] = None) -> dict:
        """One step (alodlm_denoise_step); sample=(seed, step) draws the committed tokens
        (alodlm_denoise_step_sampled)."""
        B, N = block_ids.shape
        if out is None:
            out = self.alloc_outputs(B, N, k_max)
        so = StepOut(**{k: _ptr(v) for k, v in out.items()})
        self._order_in()
        if sample is None:
            rc = lib().alodlm_denoise_step(self._h, _ptr(block_ids), B, N, float(tau_H), float(lam), k_max, rule,
                                           ctypes.byref(so))
        else:
            rc = lib().alodlm_denoise_step_sampled(self._h, _ptr(block_ids), B, N, float(tau_H), float(lam), k_max,
                                                   rule, int(sample[0]), int(sample[1]), ctypes.byref(so))
        self._check(rc, "denoise_step")
        self._order_out()
        self.N = N
        return out

    def decode_block(self, block_ids: torch.Tensor, tau_H: float, lam: float, k_max: int, rule: int = RULE_PAPER,
                     max_steps: int = 0, sample_seed: Optional[int] = None) -> dict:
        """Denoising steps until no [MASK] is left (alodlm_decode_block); max_steps 0 = N.
        Returns the device outputs (tokens, commit_step, commit_depth, steps_run, loops
        [S, B], rows [S, 2, K]) and "steps" (host int)."""
        B, N = block_ids.shape
        S = max_steps if max_steps > 0 else N
        i32 = dict(dtype=torch.int32, device="cuda")
        out = dict(tokens=torch.empty((B, N), **i32), commit_step=torch.empty((B, N), **i32),
                   commit_depth=torch.empty((B, N), **i32), steps_run=torch.empty((B,), **i32),
                   loops=torch.empty((S, B), **i32), rows=torch.empty((S, 2, k_max), **i32))
        do = DecodeOut(**{k: _ptr(v) for k, v in out.items()})
        steps = ctypes.c_int()
        self._order_in()
        if sample_seed is None:
            rc = lib().alodlm_decode_block(self._h, _ptr(block_ids), B, N, float(tau_H), float(lam), k_max, rule, S,
                                           ctypes.byref(do), ctypes.byref(steps))
        else:
            rc = lib().alodlm_decode_block_sampled(self._h, _ptr(block_ids), B, N, float(tau_H), float(lam), k_max,
                                                   rule, S, int(sample_seed), ctypes.byref(do), ctypes.byref(steps))
        self._check(rc, "decode_block")
        self._order_out()
        self.N = N
        out["steps"] = steps.value
        return out

    def sync(self):
        self._check(lib().alodlm_sync(self._h), "sync")

    def inject_wait_timeout(self):
        """Queue the error-path probe (a bounded wait that expires after about 2 s); the next
        sync() raises AlodlmError with ALODLM_ETIMEOUT."""
        self._check(lib().alodlm_inject_wait_timeout(self._h), "inject_wait_timeout")

    def debug_state(self, which: int, loop: int) -> torch.Tensor:
        dst = torch.empty((self.B, self.N, self.shape.hidden), dtype=torch.float32, device="cuda")
        self._order_in()
        self._check(lib().alodlm_debug_state(self._h, which, loop, _ptr(dst)), "debug_state")
        self._order_out()
        return dst

    def kv_slot(self, which: int, slot: int, b: int, n_pos: int) -> torch.Tensor:
        s = self.shape
        dst = torch.empty((s.n_kv_heads, n_pos, s.head_dim), dtype=torch.bfloat16, device="cuda")
        self._order_in()
        self._check(lib().alodlm_kv_slot(self._h, which, slot, b, n_pos, _ptr(dst)), "kv_slot")
        self._order_out()
        return dst

    def set_timing(self, on: bool):
        self._check(lib().alodlm_set_timing(self._h, int(on)), "set_timing")

    def set_graphs(self, on: bool):
        self._check(lib().alodlm_set_graphs(self._h, int(on)), "set_graphs")

    def step_stats(self) -> dict:
        n = ctypes.c_int()
        t = (ctypes.c_double * N_KCLASS)()
        c = (ctypes.c_int * N_KCLASS)()
        by = (ctypes.c_double * N_KCLASS)()
        fl = (ctypes.c_double * N_KCLASS)()
        self._check(lib().alodlm_step_stats(self._h, ctypes.byref(n), t, c, by, fl), "step_stats")
        names = [lib().alodlm_kernel_class_name(i).decode() for i in range(N_KCLASS)]
        return dict(launches=n.value,
                    classes={names[i]: dict(ms=t[i], launches=c[i], bytes=by[i], flops=fl[i])
                             for i in range(N_KCLASS)})


def slot_core(shape, k_max: int, c: int, d: int) -> int:
    return shape.n_prelude + (d - 1) * shape.n_core + c


def slot_coda(shape, k_max: int, j: int) -> int:
    return shape.n_prelude + k_max * shape.n_core + j
