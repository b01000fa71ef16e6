"""Host-side checks of the C ABI: the library loads, exports every function
that include/attn.h declares, and rejects bad arguments before any launch.
No test here runs a kernel, so the file needs no GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    import exact_tiled_attention_softmax_b200 as eta
    if not os.path.exists(eta.library_path()):
        from exact_tiled_attention_softmax_b200 import build
        build.build()
    return eta.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"attn_fwd", "attn_bwd", "attn_fwd_workspace_size", "attn_bwd_workspace_size",
            "attn_get_status", "attn_status_string", "attn_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    text = open(HEADER).read()
    ver = int(re.search(r"#define ATTN_VERSION (\d+)", text).group(1))
    assert lib.attn_version() == ver
    for code in range(6):
        assert lib.attn_status_string(code)
    assert b"unknown" in lib.attn_status_string(99)


def _t(shape, dtype=1, data=0x1000, stride=None):
    import exact_tiled_attention_softmax_b200 as eta
    c = eta.AttnTensorC()
    c.data = data
    c.dtype = dtype
    c.ndim = len(shape)
    st = [1] * len(shape)
    for i in range(len(shape) - 2, -1, -1):
        st[i] = st[i + 1] * shape[i + 1]
    for i, n in enumerate(shape):
        c.shape[i] = n
        c.stride[i] = (stride or st)[i]
    return c


def _call_fwd(lib, q, k, v, o, lse, mask=None, ws=0x100000, ws_bytes=1 << 20, scale=0.1):
    return lib.attn_fwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v),
                        ctypes.byref(mask) if mask else None, ctypes.c_float(scale),
                        ctypes.byref(o), ctypes.byref(lse), ws, ws_bytes, None)


def test_invalid_arguments_rejected_on_host(lib):
    import exact_tiled_attention_softmax_b200 as eta
    q, k, v = _t([1, 4, 64, 128]), _t([1, 2, 64, 128]), _t([1, 2, 64, 128])
    o, lse = _t([1, 4, 64, 128]), _t([1, 4, 64], dtype=0)
    # Hq not a multiple of Hkv
    assert _call_fwd(lib, q, _t([1, 3, 64, 128]), _t([1, 3, 64, 128]), o, lse) == eta.ATTN_ERR_INVALID_ARG
    # K and V lengths differ
    assert _call_fwd(lib, q, _t([1, 2, 65, 128]), v, o, lse) == eta.ATTN_ERR_INVALID_ARG
    # inner stride not 1
    assert _call_fwd(lib, _t([1, 4, 64, 128], stride=[64 * 256, 64 * 256, 256, 2]), k, v, o,
                     lse) == eta.ATTN_ERR_INVALID_ARG
    # mixed dtypes
    assert _call_fwd(lib, q, _t([1, 2, 64, 128], dtype=0), v, o, lse) == eta.ATTN_ERR_INVALID_ARG
    # lse must be fp32
    assert _call_fwd(lib, q, k, v, o, _t([1, 4, 64], dtype=1)) == eta.ATTN_ERR_INVALID_ARG
    # head width beyond the kernels
    big = _t([1, 4, 64, 640])
    assert _call_fwd(lib, big, _t([1, 2, 64, 640]), v, o, lse) == eta.ATTN_ERR_UNSUPPORTED
    # dropout rate outside [0, 1)
    m = eta.AllowedSet(causal=True, dropout_p=1.0).to_c()
    assert _call_fwd(lib, q, k, v, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    # window without a width
    m = eta.AttnMaskC()
    m.flags = eta.ATTN_MASK_WINDOW
    assert _call_fwd(lib, q, k, v, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    # unknown flag bits
    m.flags = 0x100
    assert _call_fwd(lib, q, k, v, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    # unknown LSE format bits
    m = eta.AttnMaskC()
    m.lse_format = 0x4
    assert _call_fwd(lib, q, k, v, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    # active lengths: a pointer is required, and Tq must equal Tk
    m = eta.AttnMaskC()
    m.flags = eta.ATTN_MASK_LENGTHS
    assert _call_fwd(lib, q, k, v, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    m.lengths = 0x4000
    k2, v2 = _t([1, 2, 96, 128]), _t([1, 2, 96, 128])
    assert _call_fwd(lib, q, k2, v2, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    # per-row starts: a pointer is required and the batch stride may not be negative
    m = eta.AttnMaskC()
    m.flags = eta.ATTN_MASK_STARTS
    assert _call_fwd(lib, q, k, v, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    m.starts = 0x4000
    m.starts_stride_b = -1
    assert _call_fwd(lib, q, k, v, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    # workspace missing or too small
    assert _call_fwd(lib, q, k, v, o, lse, ws=0) == eta.ATTN_ERR_WORKSPACE
    assert _call_fwd(lib, q, k, v, o, lse, ws_bytes=16) == eta.ATTN_ERR_WORKSPACE
    assert _call_fwd(lib, q, k, v, o, lse, ws=0x100010) == eta.ATTN_ERR_WORKSPACE
    # non-finite scale
    assert _call_fwd(lib, q, k, v, o, lse, scale=float("nan")) == eta.ATTN_ERR_INVALID_ARG


def test_topk_arguments_rejected_on_host(lib):
    import exact_tiled_attention_softmax_b200 as eta
    q = _t([16, 4, 64])
    kv = _t([32, 64])
    v_ok = _t([32, 48], stride=[64, 1])
    v_bad = _t([32, 48], data=0x2000, stride=[64, 1])
    o, lse = _t([16, 4, 48]), _t([16, 4], dtype=0)
    m = eta.AttnMaskC()
    m.flags = eta.ATTN_MASK_TOPK
    m.topk_idxs = 0x3000
    m.topk_max = 8
    m.topk_stride = 8
    # V must be a view of the same KV rows
    assert _call_fwd(lib, q, kv, v_bad, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    # causal flag is carried by the lists themselves
    m.flags = eta.ATTN_MASK_TOPK | eta.ATTN_MASK_CAUSAL
    assert _call_fwd(lib, q, kv, v_ok, o, lse, mask=m) == eta.ATTN_ERR_UNSUPPORTED
    m.flags = eta.ATTN_MASK_TOPK
    m.topk_stride = 4
    assert _call_fwd(lib, q, kv, v_ok, o, lse, mask=m) == eta.ATTN_ERR_INVALID_ARG
    # row-interval layouts are dense-only
    m.topk_stride = 8
    m.flags = eta.ATTN_MASK_TOPK | eta.ATTN_MASK_STARTS
    m.starts = 0x4000
    assert _call_fwd(lib, q, kv, v_ok, o, lse, mask=m) == eta.ATTN_ERR_UNSUPPORTED
    m.flags = eta.ATTN_MASK_TOPK
    # Dv larger than Dqk
    assert _call_fwd(lib, q, kv, _t([32, 80], stride=[64, 1]), _t([16, 4, 80]), lse,
                     mask=m) == eta.ATTN_ERR_INVALID_ARG


def test_workspace_sizes_cover_scratch(lib):
    import exact_tiled_attention_softmax_b200 as eta
    q, k, v = _t([2, 8, 256, 64]), _t([2, 4, 256, 64]), _t([2, 4, 256, 64])
    f = lib.attn_fwd_workspace_size(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), None)
    b = lib.attn_bwd_workspace_size(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), None)
    rows = 2 * 8 * 256
    assert f >= 256 and f % 256 == 0
    assert b >= 256 + rows * 4 + rows * 64 * 4
    m = eta.AttnMaskC()
    m.flags = eta.ATTN_MASK_TOPK
    m.topk_idxs = 0x3000
    m.topk_max = m.topk_stride = 8
    qt, kv, vt = _t([16, 4, 64]), _t([32, 64]), _t([32, 48], stride=[64, 1])
    bt = lib.attn_bwd_workspace_size(ctypes.byref(qt), ctypes.byref(kv), ctypes.byref(vt), ctypes.byref(m))
    assert bt >= 256 + 16 * 4 * 4 + 32 * 64 * 8


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes mirrors of attn_tensor and attn_mask have the C layout:
    a host C program built against the header prints each field's offset."""
    import shutil
    import subprocess
    import exact_tiled_attention_softmax_b200 as eta
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    structs = {"attn_tensor": eta.AttnTensorC, "attn_mask": eta.AttnMaskC}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "attn.h"', "int main(void) {"]
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {tuple(line.split()[:2]): int(line.split()[2]) for line in out if line}
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def test_fp16_lse_formats_and_reverse_flags_on_host(lib):
    """fp16 tensors pass the dtype checks (the call stops at the workspace
    check, before any launch); a non-default LSE format adds room for the
    reverse pass's natural-log copy; unknown reverse flags are rejected."""
    import exact_tiled_attention_softmax_b200 as eta
    q, k, v = _t([1, 4, 64, 128], dtype=2), _t([1, 2, 64, 128], dtype=2), _t([1, 2, 64, 128], dtype=2)
    o, lse = _t([1, 4, 64, 128], dtype=2), _t([1, 4, 64], dtype=0)
    assert _call_fwd(lib, q, k, v, o, lse, ws_bytes=16) == eta.ATTN_ERR_WORKSPACE
    base = eta.AttnMaskC()
    base.flags = eta.ATTN_MASK_CAUSAL
    kv_only = eta.AttnMaskC()
    kv_only.flags = eta.ATTN_MASK_CAUSAL
    kv_only.lse_format = eta.ATTN_LSE_KV_ONLY
    args = (ctypes.byref(q), ctypes.byref(k), ctypes.byref(v))
    b0 = lib.attn_bwd_workspace_size(*args, ctypes.byref(base))
    b1 = lib.attn_bwd_workspace_size(*args, ctypes.byref(kv_only))
    assert b1 >= b0 + 4 * 64 * 4
    bad = eta.AttnMaskC()
    bad.bwd_flags = 0x2
    assert _call_fwd(lib, q, k, v, o, lse, mask=bad) == eta.ATTN_ERR_INVALID_ARG
    det = eta.AttnMaskC()
    det.bwd_flags = eta.ATTN_BWD_DETERMINISTIC
    assert _call_fwd(lib, q, k, v, o, lse, mask=det, ws_bytes=16) == eta.ATTN_ERR_WORKSPACE


def test_selftest_rejects_bad_workspace_on_host(lib):
    import exact_tiled_attention_softmax_b200 as eta
    # Each is refused before any CUDA call is made.
    assert lib.attn_selftest_wait_timeout(None, 256, None) == eta.ATTN_ERR_WORKSPACE
    assert lib.attn_selftest_wait_timeout(0x100000, 128, None) == eta.ATTN_ERR_WORKSPACE
    assert lib.attn_selftest_wait_timeout(0x100010, 256, None) == eta.ATTN_ERR_WORKSPACE


def test_binding_checks_mask_tensors_before_the_library_sees_them(lib):
    import torch

    import exact_tiled_attention_softmax_b200 as eta
    ok_bm = torch.ones(4, 4, dtype=torch.uint8)
    eta.AllowedSet(block_mask=ok_bm).to_c()
    eta.AllowedSet(block_mask=ok_bm.bool()[None, None]).to_c()
    bad = [
        dict(block_mask=ok_bm[None]),                               # 3-D grid would be misread
        dict(block_mask=ok_bm.to(torch.int32)),
        dict(block_mask=ok_bm.t().contiguous().t()),                # columns not contiguous
        dict(topk_idxs=torch.zeros(4, 8, dtype=torch.int64)),
        dict(topk_idxs=torch.zeros(4, 8, dtype=torch.int32), topk_length=torch.zeros(4, dtype=torch.int64)),
        dict(sink=torch.zeros(4, dtype=torch.float64)),
        dict(lengths=torch.zeros(2, 1, dtype=torch.int32)),
        dict(starts=torch.zeros(2, 3, 4, dtype=torch.int32)),
    ]
    for kw in bad:
        with pytest.raises(ValueError):
            eta.AllowedSet(**kw).to_c()


def test_binding_refuses_host_tensors(lib):
    import torch

    import exact_tiled_attention_softmax_b200 as eta
    q = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        eta.attn_fwd(q, q, q, eta.AllowedSet(causal=True), 0.1)
    with pytest.raises(ValueError, match="CUDA"):
        eta.attn_bwd(q, q, q, q, q, torch.zeros(1, 2, 8), None, 0.1)


def test_a_plain_c_program_links_and_calls_the_library(lib, tmp_path):
    """tests/c_abi_caller.c links against libattn.so with no Python in
    between; its workspace sizes equal the ctypes calls' and the library
    refuses its bad call on the host."""
    import shutil
    import subprocess
    import exact_tiled_attention_softmax_b200 as eta
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    libdir = os.path.dirname(eta.library_path())
    cuda_lib = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "lib64")
    exe = tmp_path / "caller"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_caller.c"), "-o", str(exe),
                    "-L", libdir, "-l:libattn.so", f"-Wl,-rpath,{libdir}", "-L", cuda_lib,
                    f"-Wl,-rpath-link,{cuda_lib}"], check=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, run.stdout + run.stderr
    words = run.stdout.split()
    q, k, v = _t([1, 4, 300, 128]), _t([1, 2, 300, 128]), _t([1, 2, 300, 128])
    m = eta.AllowedSet(causal=True).to_c()
    refs = [ctypes.byref(x) for x in (q, k, v, m)]
    assert int(words[1]) == lib.attn_fwd_workspace_size(*refs)
    assert int(words[3]) == lib.attn_bwd_workspace_size(*refs)
    assert int(words[5]) == eta.ATTN_ERR_INVALID_ARG
