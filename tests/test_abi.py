"""The C ABI library: it loads, exports every declared entry point, sizes its
workspace, and rejects bad arguments before touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lwm_attn.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lwm_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lwm():
    from long_context_causal_attention_b200 import build
    build.build()
    import long_context_causal_attention_b200 as m
    return m


def test_library_exports_every_declared_symbol(lwm):
    declared = _declared_functions()
    assert set(declared) >= {"lwm_attn_fwd", "lwm_attn_bwd", "lwm_rope_apply",
                             "lwm_attn_workspace_size", "lwm_attn_read_status",
                             "lwm_status_string"}
    lib = ctypes.CDLL(lwm.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) <= set(lwm.ENTRY_POINTS)


def test_desc_struct_matches_header_layout(lwm):
    d = lwm.LwmAttnDesc
    assert ctypes.sizeof(d) == 64
    assert d.rope_theta.offset == 40 and d.softmax_scale.offset == 48
    assert d.segment_ids.offset == 56


def _desc(lwm, **kw):
    base = dict(batch=2, seqlen=300, heads=4, head_dim=128, dtype=0, causal=1,
                rope_theta=1e6, softmax_scale=0.0, segment_ids=None)
    base.update(kw)
    return lwm.LwmAttnDesc(**base)


def test_workspace_size(lwm):
    d = _desc(lwm)
    f = lwm.lwm_attn_workspace_size(d, False)
    b = lwm.lwm_attn_workspace_size(d, True)
    nel = 2 * 300 * 4 * 128
    assert f >= 2 * nel * 2 and b >= f
    assert f % 1024 == 0 and b % 1024 == 0
    # no rotation: the rotated copies are not needed
    assert lwm.lwm_attn_workspace_size(_desc(lwm, rope_theta=0.0), False) < f
    assert lwm.lwm_attn_workspace_size(_desc(lwm, head_dim=96), False) == 0
    assert lwm.lwm_attn_workspace_size(_desc(lwm, dtype=7), True) == 0


def test_status_strings(lwm):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lwm.lwm_status_string(code).startswith("LWM_")
    assert "unknown" in lwm.lwm_status_string(42)


def test_argument_errors_return_before_any_launch(lwm):
    lib = lwm._lib.lib()
    P = 0x10000  # fake, aligned, never dereferenced: every check below fails first
    big = 1 << 40
    d = _desc(lwm)
    args = lambda desc, ws=P, wsb=big, q=P: (ctypes.byref(desc), q, P, P, P, P, ws, wsb, None)
    assert lib.lwm_attn_fwd(None, P, P, P, P, P, P, big, None) == -1
    assert lib.lwm_attn_fwd(*args(_desc(lwm, head_dim=96))) == -2
    assert lib.lwm_attn_fwd(*args(_desc(lwm, dtype=3))) == -1
    assert lib.lwm_attn_fwd(*args(_desc(lwm, causal=2))) == -1
    assert lib.lwm_attn_fwd(*args(_desc(lwm, rope_theta=float("nan")))) == -1
    assert lib.lwm_attn_fwd(*args(d, q=None)) == -1
    assert lib.lwm_attn_fwd(*args(d, q=P + 8)) == -3
    assert lib.lwm_attn_fwd(*args(d, ws=None)) == -4
    assert lib.lwm_attn_fwd(*args(d, wsb=1024)) == -4
    assert lib.lwm_attn_fwd(*args(d, ws=P + 16)) == -3
    assert lib.lwm_attn_fwd(*args(_desc(lwm, heads=0))) == -1
    assert lib.lwm_attn_fwd(*args(_desc(lwm, segment_ids=P + 2))) == -3
    # empty problems are a successful no-op
    assert lib.lwm_attn_fwd(*args(_desc(lwm, seqlen=0))) == 0
    assert lib.lwm_attn_fwd(*args(_desc(lwm, batch=0))) == 0
    bw = lambda desc, ws=P, wsb=big: (ctypes.byref(desc), P, P, P, P, P, P, P, P, P, ws, wsb, None)
    assert lib.lwm_attn_bwd(*bw(d, wsb=lwm.lwm_attn_workspace_size(d, False) - 1)) == -4
    assert lib.lwm_attn_bwd(*bw(_desc(lwm, head_dim=32))) == -2
    assert lib.lwm_rope_apply(1, 8, 2, 7, 0, 1e4, P, P, 0, None) == -1
    assert lib.lwm_rope_apply(1, 8, 2, 12, 0, 1e4, P, P, 0, None) == -2
    assert lib.lwm_rope_apply(1, 8, 2, 64, 0, 1e4, P + 4, P, 0, None) == -3
    assert lib.lwm_rope_apply(0, 8, 2, 64, 0, 1e4, None, None, 0, None) == 0
    assert lib.lwm_attn_read_status(None, None) == -1


def test_decode_workspace_and_argument_errors(lwm):
    """Decode entry point: sizes and every refusal that happens before a launch."""
    lib = lwm._lib.lib()
    P = 0x10000
    big = 1 << 40
    d = _desc(lwm)  # B2 S300 H4 D128 bf16
    ws1 = lwm.lwm_attn_decode_workspace_size(d, 1)
    ws4 = lwm.lwm_attn_decode_workspace_size(d, 4)
    chunks = (300 + 511) // 512
    assert ws1 >= 2 * 4 * chunks * 130 * 4 and ws4 > ws1 and ws4 % 1024 == 0
    assert lwm.lwm_attn_decode_workspace_size(d, 0) == 0
    assert lwm.lwm_attn_decode_workspace_size(d, 301) == 0
    dec = lambda desc, n=1, q=P, ws=P, wsb=big: (ctypes.byref(desc), n, q, P, P, P, P, ws, wsb, None)
    assert lib.lwm_attn_decode(*dec(_desc(lwm, dtype=1))) == -2       # fp32
    assert lib.lwm_attn_decode(*dec(_desc(lwm, head_dim=64))) == -2   # D = 64
    assert lib.lwm_attn_decode(*dec(d, n=0)) == -1
    assert lib.lwm_attn_decode(*dec(d, n=301)) == -1
    assert lib.lwm_attn_decode(*dec(d, n=17)) == -2                   # above the maximum
    assert lib.lwm_attn_decode(*dec(d, q=None)) == -1
    assert lib.lwm_attn_decode(*dec(d, q=P + 8)) == -3
    assert lib.lwm_attn_decode(*dec(d, ws=None)) == -4
    assert lib.lwm_attn_decode(*dec(d, wsb=ws1 - 1)) == -4
    assert lib.lwm_attn_decode(*dec(d, ws=P + 16)) == -3
    assert lib.lwm_attn_decode(*dec(_desc(lwm, batch=0))) == 0


def test_ring_entry_points_reject_bad_arguments(lwm):
    lib = lwm._lib.lib()
    P = 0x10000
    assert lib.lwm_rope_apply_at(1, 8, 2, 64, 0, 1e4, -1, P, P, 0, None) == -1  # negative offset
    assert lib.lwm_rope_apply_at(1, 8, 2, 64, 0, 1e4, 5, P + 4, P, 0, None) == -3
    assert lib.lwm_rope_apply_at(0, 8, 2, 64, 0, 1e4, 5, None, None, 0, None) == 0
    assert lib.lwm_attn_merge(1, 8, 2, 64, 5, P, P, P, P, None) == -1            # dtype
    assert lib.lwm_attn_merge(1, 8, 2, 64, 0, None, P, P, P, None) == -1
    assert lib.lwm_attn_merge(0, 8, 2, 64, 0, None, None, None, None, None) == 0
    assert lib.lwm_accumulate(-1, 0, P, P, None) == -1
    assert lib.lwm_accumulate(0, 0, None, None, None) == 0
    assert lib.lwm_convert_f32(4, 2, P, P, None) == -1
    assert lib.lwm_convert_f32(4, 0, None, P, None) == -1


def test_pair_entry_points_need_both_or_neither_segment_arrays(lwm):
    lib = lwm._lib.lib()
    P = 0x10000
    big = 1 << 40
    with_ids = _desc(lwm, segment_ids=P)
    no_ids = _desc(lwm)
    fwd = lambda d, kseg: lib.lwm_attn_fwd_pair(ctypes.byref(d), kseg, P, P, P, P, P, P, big, None)
    assert fwd(with_ids, None) == -1
    assert fwd(no_ids, P) == -1
    assert fwd(with_ids, P + 2) == -3
    bwd = lambda d, kseg: lib.lwm_attn_bwd_pair(ctypes.byref(d), kseg, P, P, P, P, P, P, P, P, P,
                                                P, big, None)
    assert bwd(with_ids, None) == -1
    assert bwd(_desc(lwm, head_dim=32, segment_ids=P), P) == -2


def test_packed_cross_entropy_argument_errors(lwm):
    lib = lwm._lib.lib()
    P = 0x10000
    ws = lwm._lib.lib().lwm_packed_ce_workspace_size(2, 100)
    assert ws >= 2 * 100 * 8
    ce = lambda V, dt=0, logits=P, ws_b=1 << 30: lib.lwm_packed_cross_entropy(
        2, 100, V, dt, logits, P, None, P, P, P, ws_b, None)
    assert ce(40000) == -2            # row does not fit the registers of one CTA
    assert ce(20000, dt=1) == -2
    assert ce(1001) == -2             # bf16 rows must be whole 16-byte vectors
    assert ce(1000, dt=5) == -1
    assert ce(1000, logits=P + 8) == -3
    assert ce(1000, ws_b=16) == -4


def test_python_binding_requires_cuda_tensors(lwm):
    import torch
    q = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError):
        lwm.lwm_attn_fwd(q, q, q)


C_CONSUMER = r"""
#include <stdio.h>
#include <string.h>
#include "lwm_attn.h"

int main(void) {
  lwm_attn_desc d;
  memset(&d, 0, sizeof d);
  d.batch = 2; d.seqlen = 300; d.heads = 4; d.head_dim = 128;
  d.dtype = LWM_DTYPE_BF16; d.causal = 1; d.rope_theta = 1e6; d.softmax_scale = 0.0f;
  d.segment_ids = NULL;
  size_t f = lwm_attn_workspace_size(&d, 0), b = lwm_attn_workspace_size(&d, 1);
  lwm_status s = lwm_attn_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  printf("%zu %zu %d %s %s\n", f, b, (int)s, lwm_status_string(LWM_OK),
         lwm_status_string(LWM_ERR_INVALID_ARG));
  return 0;
}
"""


def test_c_program_compiles_against_the_header_and_links(lwm, tmp_path):
    """The boundary is plain C: a C11 program includes the header, links the
    library and gets the same answers as the binding (no GPU touched)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(lwm.LIB_PATH)
    subprocess.run([cc, "-std=c11", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-llwm_attn", "-Wl,-rpath," + libdir],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    d = _desc(lwm)
    assert int(out[0]) == lwm.lwm_attn_workspace_size(d, False)
    assert int(out[1]) == lwm.lwm_attn_workspace_size(d, True)
    assert int(out[2]) == -1
    assert out[3] == "LWM_OK" and out[4].startswith("LWM_ERR_INVALID")
