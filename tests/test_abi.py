"""The C ABI: the library loads without a GPU, exports every declared entry
point, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    for n in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer",
              "moe_workspace_size", "moe_pack_weights", "moe_get_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import routed_expert_ffn_05_b200 as M
    for n in declared_functions():
        assert hasattr(M.lib, n), n
        assert hasattr(M, n) or n == "moe_status_string", n


def test_library_exports_nothing_undeclared():
    # the shared object's dynamic symbol table holds exactly the header's entry points
    import subprocess
    import routed_expert_ffn_05_b200 as M
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("nm unavailable")
    exported = {l.split()[-1] for l in out.stdout.splitlines() if " T " in l}
    assert exported == set(declared_functions()), sorted(exported ^ set(declared_functions()))


def test_host_side_argument_checks():
    import routed_expert_ffn_05_b200 as M
    d = M.make_dims(4, 4096, 2048, 256, 8)
    assert M.moe_workspace_size(d) > 0
    assert M.moe_packed_size(d, M.MOE_MAT_W1) >= 256 * 2048 * 4096 * 17 // 32
    bad = [M.make_dims(4, 4000, 2048, 256, 8), M.make_dims(4, 4096, 2048, 256, 300),
           M.make_dims(4, 4096, 2048, 4, 8), M.make_dims(-1, 4096, 2048, 256, 8),
           M.make_dims(4, 4096, 2048, 256, 8, route=7)]
    for b in bad:
        with pytest.raises(M.MoeError) as ei:
            M.moe_workspace_size(b)
        assert ei.value.status == M.MOE_ERR_INVALID_ARG
    w = M.make_weights(None, None, None)
    with pytest.raises(M.MoeError) as ei:  # NULL routed weights: rejected before any launch
        M.moe_layer(d, w, 0x1000, None, 0x1000, 0x1000, stream=0)
    assert ei.value.status == M.MOE_ERR_INVALID_ARG
    with pytest.raises(M.MoeError):        # misaligned workspace
        M.moe_permute(d, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1001, stream=0)
    with pytest.raises(M.MoeError):        # hash routing without token ids
        M.moe_route(M.make_dims(4, 4096, 2048, 256, 8, route=M.MOE_ROUTE_HASH), 0x1000, w, None,
                    0x1000, 0x1000, 0x1000, stream=0)
    assert M.status_string(M.MOE_ERR_DEVICE) == "device error word set"


def header_constants():
    """Every `MOE_NAME = value` an enum of the header defines."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for body in re.findall(r"enum\s*\{(.*?)\}", src, flags=re.S):
        for name, val in re.findall(r"(MOE_\w+)\s*=\s*(\d+)", body):
            out[name] = int(val)
    return out


def header_struct_fields(name):
    """Field names of `typedef struct { ... } name;` in declaration order."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    body = re.search(r"typedef struct\s*\{([^}]*)\}\s*" + name + r"\s*;", src).group(1)
    fields = []
    for decl in body.split(";"):
        for part in decl.split(","):
            words = re.findall(r"\w+", part)
            if words:
                fields.append(words[-1])
    return fields


def test_binding_constants_match_the_header():
    import routed_expert_ffn_05_b200 as M
    consts = header_constants()
    assert len(consts) >= 20
    for name, val in consts.items():
        assert getattr(M, name) == val, name


def test_binding_structs_match_the_header():
    import routed_expert_ffn_05_b200 as M
    assert [f for f, _ in M.moe_dims._fields_] == header_struct_fields("moe_dims")
    assert [f for f, _ in M.moe_weights._fields_] == header_struct_fields("moe_weights")
    assert [f for f, _ in M.moe_cache_stats._fields_] == header_struct_fields("moe_cache_stats")


def test_static_ws_bound_matches_its_documentation():
    """The header says moe_layer_static_ws holds T = 97 decode tokens (d_model
    4096, d_ff 2048, E 256, k 8, shared d_ff 2048): the workspace of T = 97
    fits the built-in array and that of T = 98 does not."""
    import routed_expert_ffn_05_b200 as M
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    mib = int(re.search(r"#define MOE_STATIC_WS_BYTES \((\d+)u << 20\)", src).group(1))
    assert M.MOE_STATIC_WS_BYTES == mib << 20
    documented = int(re.search(r"holds up to T = (\d+) tokens", src).group(1))
    ws = lambda T: M.moe_workspace_size(M.make_dims(T, 4096, 2048, 256, 8, d_ff_shared=2048))
    assert ws(documented) <= M.MOE_STATIC_WS_BYTES < ws(documented + 1)
