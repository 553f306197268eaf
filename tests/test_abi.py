"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry
point the header declares, its structs match the Python binding's layout, and argument
validation fails cleanly before any device work."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "alodlm.h")


@pytest.fixture(scope="module")
def L():
    from adaptively_looped_masked_b200.build import build
    build()
    import adaptively_looped_masked_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ALODLM_API\s+[\w\s\*]*?\b(alodlm_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("alodlm_create", "alodlm_prefill", "alodlm_denoise_step", "alodlm_sync", "alodlm_destroy",
                     "alodlm_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    lib = L.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (alodlm_\w+)", out))
    assert exported == set(declared_functions())


LAYOUT_C = r"""
#include <stdio.h>
#include <stddef.h>
#include "alodlm.h"
#define P(T, f) printf(#T "." #f " %zu\n", offsetof(T, f))
int main(void) {
  printf("alodlm_cfg %zu\nalodlm_layer_w %zu\nalodlm_weights %zu\nalodlm_step_out %zu\n",
         sizeof(alodlm_cfg), sizeof(alodlm_layer_w), sizeof(alodlm_weights), sizeof(alodlm_step_out));
  P(alodlm_cfg, rope_base); P(alodlm_cfg, mask_id); P(alodlm_cfg, mem_limit_bytes); P(alodlm_cfg, debug_dump);
  P(alodlm_weights, exit_b); P(alodlm_weights, layers); P(alodlm_step_out, readout_rows);
  printf("alodlm_decode_out %zu\n", sizeof(alodlm_decode_out)); P(alodlm_decode_out, rows);
  return 0;
}
"""


def test_struct_layout_matches_binding(L):
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "l.c"), os.path.join(d, "l")
        open(src, "w").write(LAYOUT_C)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True)
        got = dict(line.rsplit(" ", 1) for line in subprocess.run([exe], capture_output=True, text=True,
                                                                  check=True).stdout.split("\n") if line)
    got = {k: int(v) for k, v in got.items()}
    assert got["alodlm_cfg"] == ctypes.sizeof(L.Cfg)
    assert got["alodlm_layer_w"] == ctypes.sizeof(L.LayerW)
    assert got["alodlm_weights"] == ctypes.sizeof(L.Weights)
    assert got["alodlm_step_out"] == ctypes.sizeof(L.StepOut)
    assert got["alodlm_cfg.rope_base"] == L.Cfg.rope_base.offset
    assert got["alodlm_cfg.mask_id"] == L.Cfg.mask_id.offset
    assert got["alodlm_cfg.mem_limit_bytes"] == L.Cfg.mem_limit_bytes.offset
    assert got["alodlm_cfg.debug_dump"] == L.Cfg.debug_dump.offset
    assert got["alodlm_weights.exit_b"] == L.Weights.exit_b.offset
    assert got["alodlm_weights.layers"] == L.Weights.layers.offset
    assert got["alodlm_step_out.readout_rows"] == L.StepOut.readout_rows.offset
    assert got["alodlm_decode_out"] == ctypes.sizeof(L.DecodeOut)
    assert got["alodlm_decode_out.rows"] == L.DecodeOut.rows.offset


def _cfg(L, **kw):
    base = dict(hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, inter=688, vocab=2048, n_prelude=1, n_core=2,
                n_coda=1, k_max=4, max_batch=1, max_prefix=48, max_block=16, rope_base=1e6, rms_eps=1e-6,
                mask_id=2047, qk_norm=1, mem_limit_bytes=0, debug_dump=0)
    base.update(kw)
    return L.Cfg(**base)


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(n_q_heads=3), dict(inter=100), dict(k_max=0),
                                 dict(max_block=2000), dict(mask_id=5000), dict(hidden=40), dict(n_core=0)])
def test_create_rejects_bad_config_before_device_work(L, bad):
    lib = L.lib()
    cfg = _cfg(L, **bad)
    layers = (L.LayerW * 4)()
    for i in range(4):
        for f in L.LAYER_FIELDS:
            setattr(layers[i], f, 16)
    w = L.Weights(matrix_dtype=0, embed=16, lm_head=16, final_norm=16, exit_w=16, exit_b=-1.0, layers=layers)
    h = ctypes.c_void_p()
    rc = lib.alodlm_create(ctypes.byref(cfg), ctypes.byref(w), None, ctypes.byref(h))
    assert rc == -1 and not h.value
    assert lib.alodlm_last_error(None)


def test_null_arguments_are_rejected(L):
    lib = L.lib()
    h = ctypes.c_void_p()
    assert lib.alodlm_create(None, None, None, ctypes.byref(h)) == -1
    assert lib.alodlm_prefill(None, None, 1, 1, None) == -1
    assert lib.alodlm_append(None, None, 1, 1, None) == -1
    assert lib.alodlm_denoise_step_sampled(None, None, 1, 1, 0.5, 0.5, 1, 0, 1, 1, None) == -1
    assert lib.alodlm_decode_block_sampled(None, None, 1, 1, 0.5, 0.5, 1, 0, 1, 1, None, None) == -1
    assert lib.alodlm_denoise_step(None, None, 1, 1, 0.5, 0.5, 1, 0, None) == -1
    assert lib.alodlm_decode_block(None, None, 1, 1, 0.5, 0.5, 1, 0, 1, None, None) == -1
    assert lib.alodlm_sync(None) == -1
    assert lib.alodlm_inject_wait_timeout(None) == -1
    lib.alodlm_destroy(None)
    assert lib.alodlm_kernel_class_name(0) == b"gemm"
    assert lib.alodlm_kernel_class_name(8) == b"gemm_tile"
    assert lib.alodlm_gemm_bf16(None, None, None, 1, 1, 8, None, 0, None) == -1


LINK_C = r"""
#include <stdio.h>
#include "alodlm.h"
int main(void) {
  alodlm_t *h = (alodlm_t *)1;
  alodlm_cfg cfg = {0};            /* hidden 0: rejected before any device work */
  int rc = alodlm_create(&cfg, NULL, NULL, &h);
  printf("%d %d %s\n", rc, h == NULL, alodlm_last_error(NULL) ? "msg" : "none");
  printf("%d\n", alodlm_denoise_step(NULL, NULL, 1, 1, 0.5f, 0.5f, 1, ALODLM_RULE_PAPER, NULL));
  printf("%s\n", alodlm_kernel_class_name(1));
  int32_t g[4], a[5];          /* launch partitions: pure queries, callable without a GPU */
  rc = alodlm_plan_gemm(32, 4096, 2112, g);
  printf("%d %d %d %d %d\n", rc, g[0], g[1], g[2], g[3]);
  rc = alodlm_plan_attention(128, 8, 1, 1056, 0, 148, 1, 0, a);
  printf("%d %d %d %d %d\n", rc, a[0], a[2], a[3], a[4]);
  printf("%d\n", alodlm_plan_gemm(32, 4096, 2112, NULL));
  alodlm_destroy(NULL);
  return 0;
}
"""


def test_plain_c_program_links_and_calls_the_library(L):
    """The boundary is plain C: a C program compiled with gcc against include/alodlm.h links
    libalodlm.so and gets clean errors (no GPU needed for argument validation)."""
    lib_dir = os.path.dirname(L.LIB_PATH)
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "c.c"), os.path.join(d, "c")
        open(src, "w").write(LINK_C)
        subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), src, "-o", exe, "-L", lib_dir,
                        "-l:libalodlm.so", f"-Wl,-rpath,{lib_dir}"], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    assert out[0] == "-1 1 msg"
    assert out[1] == "-1"
    assert out[2] == "attention"
    assert out[3] == "0 32 4 9 33"   # 33 k-tiles over 4 ranks of 9
    assert out[4] == "0 1 8 128 1"   # one query tile, 8 key splits of one tile, remainder on the last
    assert out[5] == "-1"
