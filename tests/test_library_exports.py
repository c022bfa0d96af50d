"""CPU checks of the C ABI library: it loads and exports every entry point the
header declares (no compute call: there is no GPU here), and the binding's list
matches the header."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]
LIB = os.path.join(ROOT, "dynamic_short_convolutions_b200", "libdynconv.so")


def _declared():
    text = "\n".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"DYNCONV_API\s+[\w\s\*]*?\b(dynconv_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = _declared()
    for n in ("dynconv_fwd", "dynconv_fwd_varlen", "dynconv_bwd", "dynconv_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol():
    if not os.path.exists(LIB):
        from dynamic_short_convolutions_b200 import build

        build.build()
    lib = ctypes.CDLL(LIB)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    from dynamic_short_convolutions_b200 import _lib as L

    assert sorted(L.EXPORTS) == sorted(set(L.EXPORTS) & set(_declared())) or set(_declared()) >= set(L.EXPORTS)
    assert set(L.EXPORTS) == set(_declared())


def test_pure_host_entry_points_without_gpu():
    from dynamic_short_convolutions_b200 import _lib as L

    if not os.path.exists(LIB):
        pytest.skip("library not built")
    lib = L.load()
    assert lib.dynconv_version() >= 100
    assert lib.dynconv_status_string(2) == b"DYNCONV_ERR_UNSUPPORTED"
    d = L.make_desc(L.LOWRANK, L.BF16, 8, 2048, 768, 2304, 3, 32)
    assert L.dynconv_workspace_bytes(d) > 0
    assert L.dynconv_workspace_bytes(L.make_desc(L.LOWRANK, L.BF16, 8, 2048, 768, 2304, 0, 32)) == 0
    assert L.dynconv_workspace_bytes(L.make_desc(L.HEADWISE, L.BF16, 1, 10, 8, 12, 3, 0, 5)) == 0


def test_descriptor_layout_matches_header(tmp_path):
    """The ctypes descriptor has the C struct's size and field offsets (gcc on the header)."""
    import shutil
    import subprocess

    from dynamic_short_convolutions_b200 import _lib as L

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = [f[0] for f in L.dynconv_desc._fields_]
    src = tmp_path / "probe.c"
    body = "\n".join(f'    printf("{f} %zu\\n", offsetof(dynconv_desc, {f}));' for f in fields)
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "dynconv.h"\nint main(void) {\n'
                   f'    printf("size %zu\\n", sizeof(dynconv_desc));\n{body}\n    return 0;\n}}\n')
    exe = tmp_path / "probe"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                       check=True).stdout.splitlines())
    assert int(out["size"]) == ctypes.sizeof(L.dynconv_desc)
    for f in fields:
        assert int(out[f]) == getattr(L.dynconv_desc, f).offset, f


def test_channel_first_descriptor_validation():
    from dynamic_short_convolutions_b200 import _lib as L

    if not os.path.exists(LIB):
        pytest.skip("library not built")
    cf = dict(layout=L.CHANNEL_FIRST)
    ok = L.make_desc(L.LOWRANK, L.BF16, 8, 2048, 768, 2304, 3, 32, **cf)
    assert L.dynconv_workspace_bytes(ok) > 0
    # any channel stride >= seqlen (odd ones take the generic kernels); below seqlen is invalid
    assert L.dynconv_workspace_bytes(L.make_desc(L.LOWRANK, L.BF16, 2, 13, 64, 64, 3, 8, u_row_stride=15, **cf)) > 0
    assert L.dynconv_workspace_bytes(L.make_desc(L.LOWRANK, L.BF16, 2, 16, 64, 64, 3, 8, u_row_stride=15, **cf)) == 0
    assert L.dynconv_workspace_bytes(L.make_desc(L.LOWRANK, L.BF16, 2, 16, 64, 64, 3, 8, layout=2)) == 0
    # token-major keeps its 16-byte row-stride rule
    assert L.dynconv_workspace_bytes(L.make_desc(L.LOWRANK, L.BF16, 2, 16, 64, 64, 3, 8, u_row_stride=65)) == 0


def test_query_family_host_only():
    """dynconv_query_family answers without device work: a valid descriptor gets a family
    for each pass, an invalid one its validation status."""
    from dynamic_short_convolutions_b200 import _lib as L

    if not os.path.exists(LIB):
        pytest.skip("library not built")
    fwd, bwd, _ = L.dynconv_query_family(L.make_desc(L.LOWRANK, L.BF16, 8, 2048, 768, 2304, 3, 32))
    assert fwd in ("tensor_core", "cuda_core") and bwd in ("tensor_core", "cuda_core")
    fwd, bwd, why = L.dynconv_query_family(L.make_desc(L.LOWRANK, L.F32, 2, 128, 64, 64, 3, 4))
    assert (fwd, bwd) == ("cuda_core", "cuda_core") and why
    fwd, bwd, why = L.dynconv_query_family(L.make_desc(L.LOWRANK, L.BF16, 1, 64, 64, 64, 3, 16,
                                                       algo=L.ALGO_SIMT))
    assert (fwd, bwd) == ("cuda_core", "cuda_core") and "CUDA-core" in why
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_query_family(L.make_desc(L.LOWRANK, L.BF16, 1, 64, 64, 64, 5, 16))
    assert e.value.status == 2
    # a forced tensor-core run the kernels cannot do is refused, as the entry points refuse it
    with pytest.raises(L.DynConvError) as e:
        L.dynconv_query_family(L.make_desc(L.LOWRANK, L.F32, 2, 128, 64, 64, 3, 4, algo=L.ALGO_TC))
    assert e.value.status == 2 and "fp32" in str(e.value)
    # sizes whose byte counts wrap 64 bits are invalid, not small
    assert L.dynconv_workspace_bytes(L.make_desc(L.LOWRANK, L.BF16, 3, 1 << 62, 64, 64, 3, 16)) == 0
    assert "overflow" in L.dynconv_last_error()
