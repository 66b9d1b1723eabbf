"""Host-side checks of the C ABI: the library loads, exports every entry point
include/hstu.h declares, its structs match the Python binding, and argument
errors come back as status codes before anything reaches a GPU."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

from hstu_sequential_transduction_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(hstu_\w+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = ops.load_library()
    decl = declared_functions()
    assert decl, "no declarations found"
    for name in decl:
        assert hasattr(lib, name), name
    assert set(decl) <= set(ops.EXPORTED)


def test_struct_layout_matches_header(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "hstu.h"\n'
        'int main(void){printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(hstu_attn_desc),'
        ' offsetof(hstu_attn_desc,total_tokens), offsetof(hstu_attn_desc,inv_n),'
        ' offsetof(hstu_attn_desc,debug_checks), sizeof(hstu_layer_desc),'
        ' offsetof(hstu_layer_desc,ln_eps)); printf("%zu %zu\\n", offsetof(hstu_attn_desc,local_window),'
        ' offsetof(hstu_attn_desc,global_window)); printf("%zu\\n", offsetof(hstu_layer_desc,output_concat));'
        ' printf("%zu\\n", offsetof(hstu_attn_desc,fp8_qk));'
        ' printf("%zu %zu\\n", offsetof(hstu_attn_desc,cand_positions), offsetof(hstu_attn_desc,per_head_tables));'
        ' printf("%zu\\n", offsetof(hstu_layer_desc,fp8_projections)); return 0;}\n')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    D, L = ops.hstu_attn_desc, ops.hstu_layer_desc
    assert got == [ctypes.sizeof(D), D.total_tokens.offset, D.inv_n.offset, D.debug_checks.offset,
                   ctypes.sizeof(L), L.ln_eps.offset, D.local_window.offset, D.global_window.offset,
                   L.output_concat.offset, D.fp8_qk.offset, D.cand_positions.offset, D.per_head_tables.offset,
                   L.fp8_projections.offset]


def test_status_strings_and_version():
    assert ops.hstu_status_string(0) == "HSTU_OK"
    assert "WORKSPACE" in ops.hstu_status_string(3)
    assert ops.hstu_version() >= 100


def _desc(**kw):
    base = dict(num_seqs=2, max_seq_len=64, total_tokens=100, num_heads=2, d_qk=64, d_v=64,
                dtype=ops.HSTU_BF16, inv_n=1 / 64, pos_lo=-8, pos_hi=8, num_time_buckets=16)
    base.update(kw)
    return ops.make_attn_desc(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(num_heads=0), 1), (dict(num_seqs=-1), 1), (dict(pos_hi=-9), 1),
    (dict(num_time_buckets=0), 1), (dict(dtype=7), 1), (dict(d_qk=48, d_v=48), 2),
    (dict(d_v=32), 2), (dict(dtype=ops.HSTU_F32, d_qk=128, d_v=128), 2),
    (dict(inv_n=float("inf")), 1),
    # bf16 runs on the tcgen05 kernels only (head dims 64, 128); fp32 takes 32 and 64
    (dict(d_qk=32, d_v=32), 2), (dict(dtype=ops.HSTU_F32, d_qk=32, d_v=32), 0),
    (dict(d_qk=128, d_v=128), 0),
    # the two readings of the bias are switches; per-head tables must stay indexable
    (dict(cand_own_index=True, per_head_tables=True), 0),
    (dict(pos_lo=-(1 << 23), pos_hi=(1 << 23) - 1, num_heads=256, per_head_tables=True), 2),
    (dict(num_time_buckets=1 << 24, num_heads=256, per_head_tables=True), 2),
])
def test_bad_descriptors_rejected(kw, status):
    lib = ops.load_library()
    n = ctypes.c_size_t(0)
    d = _desc(**kw)
    assert lib.hstu_attn_workspace_size(ctypes.byref(d), 0, ctypes.byref(n)) == status


@pytest.mark.parametrize("field", ["cand_positions", "per_head_tables"])
def test_bias_switches_take_zero_or_one(field):
    lib = ops.load_library()
    n = ctypes.c_size_t(0)
    d = _desc()
    setattr(d, field, 2)
    assert lib.hstu_attn_workspace_size(ctypes.byref(d), 0, ctypes.byref(n)) == 1


def test_table_shapes_checked_in_binding():
    from hstu_sequential_transduction_b200.ops import _tables
    assert _tables(torch.zeros(17), torch.zeros(16), 2, -8, 8) == (16, False)
    assert _tables(torch.zeros(2, 17), torch.zeros(2, 16), 2, -8, 8) == (16, True)
    for rp, rt in ((torch.zeros(2, 17), torch.zeros(16)), (torch.zeros(3, 17), torch.zeros(3, 16)),
                   (torch.zeros(16), torch.zeros(16))):
        with pytest.raises(ValueError):
            _tables(rp, rt, 2, -8, 8)


def test_wait_test_hook_is_forward_only():
    lib = ops.load_library()
    n = ctypes.c_size_t(0)
    d = _desc()
    d.debug_checks = ops.HSTU_DEBUG_WAIT_TEST
    assert lib.hstu_attn_workspace_size(ctypes.byref(d), 0, ctypes.byref(n)) == 0
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    assert lib.hstu_attn_bwd(ctypes.byref(d), fake, fake, fake, fake, fake, None, fake, fake, fake,
                             fake, fake, fake, fake, fake, fake, ctypes.c_size_t(1 << 20), None) == 2
    layer = ops.hstu_layer_desc(d, 128, 1e-5)
    assert lib.hstu_layer_workspace_size(ctypes.byref(layer), ctypes.byref(n)) == 2
    d.debug_checks = 1  # any other value is an argument error
    assert lib.hstu_attn_workspace_size(ctypes.byref(d), 0, ctypes.byref(n)) == 1


def test_workspace_and_pointer_checks_before_launch():
    lib = ops.load_library()
    d = _desc()
    n = ctypes.c_size_t(0)
    assert lib.hstu_attn_workspace_size(ctypes.byref(d), 1, ctypes.byref(n)) == 0
    assert n.value >= 256 + 8 * (100 // 64 + 1 + 2)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    null = ctypes.c_void_p(0)
    # null seq_offsets
    assert lib.hstu_attn_fwd(ctypes.byref(d), fake, fake, fake, null, fake, null, fake, fake, fake,
                             fake, ctypes.c_size_t(n.value), null) == 1
    # misaligned q
    assert lib.hstu_attn_fwd(ctypes.byref(d), ctypes.c_void_p((1 << 20) + 2), fake, fake, fake, fake,
                             null, fake, fake, fake, fake, ctypes.c_size_t(n.value), null) == 1
    # missing / small / misaligned workspace
    assert lib.hstu_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, null, fake, fake, fake,
                             null, ctypes.c_size_t(n.value), null) == 3
    assert lib.hstu_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, null, fake, fake, fake,
                             fake, ctypes.c_size_t(16), null) == 3
    assert lib.hstu_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, null, fake, fake, fake,
                             ctypes.c_void_p((1 << 20) + 64), ctypes.c_size_t(n.value), null) == 3
    # backward: null gradient outputs
    assert lib.hstu_attn_bwd(ctypes.byref(d), fake, fake, fake, fake, fake, null, fake, fake, fake,
                             fake, fake, fake, null, fake, fake, ctypes.c_size_t(n.value), null) == 1


def test_layer_descriptor_checks():
    lib = ops.load_library()
    n = ctypes.c_size_t(0)
    ok = ops.hstu_layer_desc(_desc(num_heads=4, d_qk=128, d_v=128), 512, 1e-5)
    assert lib.hstu_layer_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == 0
    bad_width = ops.hstu_layer_desc(_desc(num_heads=3, d_qk=64, d_v=64), 512, 1e-5)
    assert lib.hstu_layer_workspace_size(ctypes.byref(bad_width), ctypes.byref(n)) == 2
    bad_d = ops.hstu_layer_desc(_desc(), 100, 1e-5)
    assert lib.hstu_layer_workspace_size(ctypes.byref(bad_d), ctypes.byref(n)) == 2
    bad_eps = ops.hstu_layer_desc(_desc(), 128, -1.0)
    assert lib.hstu_layer_workspace_size(ctypes.byref(bad_eps), ctypes.byref(n)) == 1
    plain = n.value if lib.hstu_layer_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == 0 else None
    cat = ops.hstu_layer_desc(_desc(num_heads=4, d_qk=128, d_v=128), 512, 1e-5, 1)
    assert lib.hstu_layer_workspace_size(ctypes.byref(cat), ctypes.byref(n)) == 0 and n.value == plain
    bad_cat = ops.hstu_layer_desc(_desc(num_heads=4, d_qk=128, d_v=128), 512, 1e-5, 2)
    assert lib.hstu_layer_workspace_size(ctypes.byref(bad_cat), ctypes.byref(n)) == 1


def test_library_has_no_oracle_dependency():
    # the product library and binding never reference the oracle
    pkg = os.path.join(ROOT, "hstu_sequential_transduction_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"(import\s+oracle|from\s+oracle|oracle\.|hstu_oracle|liboracle)", text), f
