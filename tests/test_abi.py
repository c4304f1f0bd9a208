"""The C-ABI library loads, exports every function include/moe.h declares, and
rejects bad arguments before touching a device.  CPU only."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import block_quantized_expert_moe_b200 as bq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_function_is_exported():
    names = declared_functions()
    assert "moe_layer_forward" in names and "moe_pack_experts" in names and "moe_route_topk" in names
    out = subprocess.run(["nm", "-D", "--defined-only", bq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (moe_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(bq.lib, n)


def test_status_strings():
    assert bq.moe_status_string(bq.MOE_OK) == "ok"
    assert "argument" in bq.moe_status_string(bq.MOE_ERR_INVALID_ARG)
    assert bq.moe_status_string(99) == "unknown status"


def test_route_workspace_size():
    assert bq.moe_route_workspace_bytes(1, 512) == 256 + 512 * 4
    assert bq.moe_route_workspace_bytes(0, 512) == 0


def _desc(**kw):
    base = dict(n_experts=4, hidden=64, inter=32, has_shared=0, max_tokens=8, max_top_k=2,
                fmt_gate_up=bq.MOE_FMT_Q8_0, fmt_down=bq.MOE_FMT_Q8_0)
    base.update(kw)
    d = bq.moe_pack_desc()
    for k, v in base.items():
        setattr(d, k, v)
    return d


@pytest.mark.parametrize("kw", [
    dict(n_experts=0), dict(n_experts=2000), dict(hidden=48), dict(inter=40), dict(max_tokens=0),
    dict(max_top_k=5), dict(fmt_gate_up=9), dict(fmt_down=0),
])
def test_pack_rejects_bad_descriptions_without_a_device(kw):
    buf = np.zeros(1 << 16, np.uint8)
    d = _desc(**kw)
    d.gate_up_blocks = buf.ctypes.data
    d.down_blocks = buf.ctypes.data
    h = ctypes.c_void_p()
    assert bq.lib.moe_pack_experts(ctypes.byref(d), 0, ctypes.byref(h)) == bq.MOE_ERR_INVALID_ARG
    assert not h.value


def test_pack_requires_tables_scales_and_shared_blocks():
    buf = np.zeros(1 << 16, np.uint8)
    for kw in (dict(fmt_gate_up=bq.MOE_FMT_IQ4_NL), dict(fmt_down=bq.MOE_FMT_NVFP4), dict(has_shared=1)):
        d = _desc(**kw)
        d.gate_up_blocks = buf.ctypes.data
        d.down_blocks = buf.ctypes.data
        h = ctypes.c_void_p()
        assert bq.lib.moe_pack_experts(ctypes.byref(d), 0, ctypes.byref(h)) == bq.MOE_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert bq.lib.moe_pack_experts(None, 0, ctypes.byref(h)) == bq.MOE_ERR_INVALID_ARG


def test_forward_and_route_reject_null_and_misaligned_pointers():
    assert bq.lib.moe_layer_forward(None, 1, None, None, 0, 1, 1, None, None) == bq.MOE_ERR_INVALID_ARG
    assert bq.lib.moe_debug_dequant_rows(None, 0, 0, 0, 1, 0, None, None) == bq.MOE_ERR_INVALID_ARG
    buf = np.zeros(4096, np.uint8)
    p = buf.ctypes.data + 8 if buf.ctypes.data % 16 == 0 else buf.ctypes.data
    assert bq.lib.moe_route_topk(p, 2, p, 1, 64, 4, 2, p, p, p, 4096, None) == bq.MOE_ERR_INVALID_ARG
    a = buf.ctypes.data + (-buf.ctypes.data % 16)
    # top_k > n_experts and hidden not a multiple of 8
    assert bq.lib.moe_route_topk(a, 2, a, 1, 64, 4, 5, a, a, a, 4096, None) == bq.MOE_ERR_INVALID_ARG
    assert bq.lib.moe_route_topk(a, 2, a, 1, 60, 4, 2, a, a, a, 4096, None) == bq.MOE_ERR_INVALID_ARG
    assert bq.lib.moe_route_topk(a, 2, a, 1, 64, 4, 2, a, a, a, 16, None) == bq.MOE_ERR_INVALID_ARG


def test_empty_batch_routes_nothing_without_a_device():
    # n_tokens == 0 is a no-op: MOE_OK before any pointer is read or any CUDA call is made
    assert bq.lib.moe_route_topk(None, 2, None, 0, 64, 4, 2, None, None, None, 0, None) == bq.MOE_OK
    assert bq.lib.moe_route_topk_noalloc(None, 1, None, 0, 64, 4, 2, None, None, None) == bq.MOE_OK
    assert bq.moe_route_workspace_bytes(0, 4) == 0
    # the other arguments are still checked, and a negative count is an error
    assert bq.lib.moe_route_topk(None, 2, None, 0, 60, 4, 2, None, None, None, 0, None) == bq.MOE_ERR_INVALID_ARG
    assert bq.lib.moe_route_topk(None, 2, None, 0, 64, 4, 5, None, None, None, 0, None) == bq.MOE_ERR_INVALID_ARG
    assert bq.lib.moe_route_topk(None, 7, None, 0, 64, 4, 2, None, None, None, 0, None) == bq.MOE_ERR_INVALID_ARG
    assert bq.lib.moe_route_topk(None, 2, None, -1, 64, 4, 2, None, None, None, 0, None) == bq.MOE_ERR_INVALID_ARG
    assert bq.lib.moe_layer_forward(None, 2, None, None, 0, 0, 1, None, None) == bq.MOE_ERR_INVALID_ARG


def test_fault_injection_entry_points_check_arguments_without_a_device():
    assert bq.lib.moe_debug_fail_alloc_after(-2) == bq.MOE_ERR_INVALID_ARG
    assert bq.lib.moe_debug_fail_alloc_after(3) == bq.MOE_OK
    assert bq.lib.moe_debug_fail_alloc_after(-1) == bq.MOE_OK
    # a pack that fails its argument checks allocates nothing, so a pending injection stays pending
    bq.moe_debug_fail_alloc_after(0)
    h = ctypes.c_void_p()
    assert bq.lib.moe_pack_experts(None, 0, ctypes.byref(h)) == bq.MOE_ERR_INVALID_ARG
    bq.moe_debug_fail_alloc_after(-1)
    assert bq.lib.moe_debug_wait_timeout(None, None) == bq.MOE_ERR_INVALID_ARG


def test_binding_rejects_bad_tensors_before_calling_the_library():
    """The C ABI sees only pointers; the binding checks what a pointer cannot carry."""
    import torch
    d = _desc(n_experts=4, hidden=64, inter=32)
    pack = bq.Pack(None, d, 0)  # never reaches the library: every call below fails its checks first
    x = torch.zeros(2, 64)
    wr = torch.zeros(4, 64, dtype=torch.int16)
    out = torch.zeros(2, 64)
    with pytest.raises(ValueError, match="CUDA"):  # host memory would reach a kernel
        bq.moe_layer_forward(x, wr, pack, 0, 2, out)
    with pytest.raises(TypeError, match="x must be"):
        bq.moe_layer_forward(x.double(), wr, pack, 0, 2, out)
    with pytest.raises(ValueError, match="router_w must have shape"):
        bq.moe_layer_forward(x, torch.zeros(5, 64, dtype=torch.int16), pack, 0, 2, out)
    with pytest.raises(ValueError, match="x must have shape"):
        bq.moe_layer_forward(torch.zeros(2, 32), wr, pack, 0, 2, out)
    with pytest.raises(ValueError, match="out must have shape"):
        bq.moe_layer_forward(x, wr, pack, 0, 2, torch.zeros(3, 64))
    with pytest.raises(TypeError, match="out must be"):
        bq.moe_layer_forward(x, wr, pack, 0, 2, out.to(torch.bfloat16))
    with pytest.raises(ValueError, match="contiguous"):
        bq.moe_layer_forward_ex(torch.zeros(64, 2).t(), wr, pack, 0, 2, out, bq.MOE_PATH_AUTO)
    with pytest.raises(ValueError, match="2-D"):
        bq.moe_layer_forward(torch.zeros(64), wr, pack, 0, 2, out)
    idx, gate = torch.zeros(2, 2, dtype=torch.int32), torch.zeros(2, 2)
    with pytest.raises(ValueError, match="CUDA"):
        bq.moe_route_topk(x, wr, 2, idx, gate, torch.zeros(4096, dtype=torch.uint8))
    with pytest.raises(TypeError, match="idx_out must be"):
        bq.moe_route_topk_noalloc(x, wr, 2, idx.long(), gate)
    with pytest.raises(ValueError, match="gate_out must have shape"):
        bq.moe_route_topk_noalloc(x, wr, 2, idx, torch.zeros(2, 3))


C_CLIENT = r"""
#include <stdio.h>
#include "moe.h"
int main(void)
{
    moe_pack *p = NULL;
    moe_status empty = moe_route_topk(NULL, MOE_DT_BF16, NULL, 0, 64, 4, 2, NULL, NULL, NULL, 0, NULL);
    moe_status bad = moe_pack_experts(NULL, 0, &p);
    printf("%s|%zu|%d|%d|%d\n", moe_status_string(MOE_ERR_INVALID_ARG), moe_route_workspace_bytes(8, 512),
           (int)empty, (int)bad, p == NULL);
    return 0;
}
"""


def test_header_compiles_as_c99_and_the_library_links_from_c(repo_tmp):
    """The boundary is a C ABI: a C99 program (warnings as errors) includes include/moe.h,
    links libmoe.so and calls it; the calls used need no device."""
    src = repo_tmp / "client.c"
    exe = repo_tmp / "client"
    src.write_text(C_CLIENT)
    libdir = os.path.dirname(bq.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lmoe", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.strip()
    assert out == f"invalid argument|{256 + 8 * 512 * 4}|{bq.MOE_OK}|{bq.MOE_ERR_INVALID_ARG}|1"


def test_python_constants_equal_the_header():
    """Every MOE_* enumerator and flag of include/moe.h has the same value in the binding."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    consts = {n: int(v) for n, v in re.findall(r"\b(MOE_[A-Z0-9_]+)\s*=\s*(\d+)", src)}
    consts.update({n: int(v) for n, v in re.findall(r"#define\s+(MOE_[A-Z0-9_]+)\s+(\d+)", src)})
    assert len(consts) >= 23, consts  # 9 statuses, 6 formats, 2 dtypes, 5 paths, 1 flag
    for name, value in consts.items():
        assert getattr(bq, name) == value, name


def test_ctypes_structures_match_the_header_layout(repo_tmp):
    """moe_pack_desc and moe_pack_info: every field at the C compiler's offset, same sizes."""
    structs = {"moe_pack_desc": bq.moe_pack_desc, "moe_pack_info": bq.moe_pack_info}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "moe.h"', "int main(void)", "{"]
    for cname, py in structs.items():
        lines.append(f'    printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in py._fields_:
            lines.append(f'    printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["    return 0;", "}"]
    src = repo_tmp / "layout.c"
    exe = repo_tmp / "layout"
    src.write_text("\n".join(lines) + "\n")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe)], check=True, capture_output=True, text=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        cname, field, value = line.split()
        got[(cname, field)] = int(value)
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for field, _ in py._fields_:
            assert got[(cname, field)] == getattr(py, field).offset, (cname, field)
