"""Host-side checks of the C ABI that need no GPU: exports, descriptor and pointer
validation, workspace and saved-buffer sizing.  No call here reaches a kernel."""
import ctypes
import os
import re
import subprocess

import pytest

from routing_grouped_gemm_route_b200 import lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"^\s*(?:moe_status|const char\*)\s+(moe_\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def L():
    from routing_grouped_gemm_route_b200 import build
    build.build()
    return lib.load()


def test_every_declared_symbol_is_exported(L):
    declared = header_symbols()
    assert len(declared) >= 17
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (moe_\w+)$", out, re.M))
    assert set(declared) <= exported, set(declared) - exported
    assert sorted(lib.EXPORTS) == declared


@pytest.mark.parametrize("args,code", [
    ((512, 128, 256, 8, 2, "fp32"), 0),
    ((16384, 2048, 1024, 128, 4, "bf16"), 0),
    ((0, 128, 64, 1, 1, "bf16"), 0),                  # no tokens is valid
    ((10, 100, 64, 8, 2, "bf16"), lib.MOE_EINVAL),    # d not a multiple of 128
    ((10, 128, 32, 8, 2, "bf16"), lib.MOE_EINVAL),    # d_ff not a multiple of 64
    ((10, 128, 64, 8, 9, "bf16"), lib.MOE_EINVAL),    # k > E
    ((10, 128, 64, 8, 0, "bf16"), lib.MOE_EINVAL),    # k < 1
    ((10, 128, 64, 1025, 2, "bf16"), lib.MOE_EINVAL), # E > 1024
    ((10, 128, 64, 64, 33, "bf16"), lib.MOE_EINVAL),  # k > 32
    ((-1, 128, 64, 8, 2, "bf16"), lib.MOE_EINVAL),
    ((2 ** 29, 128, 64, 8, 4, "bf16"), lib.MOE_EINVAL),  # T*k >= 2^31
    ((10, 128, 64, 8, 2, "mxfp8"), lib.MOE_EUNSUPPORTED),
])
def test_descriptor_checks(L, args, code):
    assert lib.moe_check_desc(lib.make_desc(*args)) == code


def test_flag_checks(L):
    assert lib.moe_check_desc(lib.make_desc(8, 128, 64, 4, 2, "bf16", 64)) == lib.MOE_EINVAL
    # the weight-code reuse is an MXFP8 option only
    keep = lib.MOE_FLAG_MX_KEEP_WEIGHT_CODES
    assert lib.moe_check_desc(lib.make_desc(8, 128, 128, 4, 2, "bf16", keep)) == lib.MOE_EINVAL
    assert lib.moe_check_desc(lib.make_desc(8, 128, 128, 4, 2, "fp32", keep)) == lib.MOE_EINVAL
    assert lib.moe_check_desc(lib.make_desc(8, 128, 128, 4, 2, "mxfp8", keep)) == 0
    assert lib.moe_check_desc(lib.make_desc(8, 128, 64, 4, 2, "bf16",
                                            lib.MOE_FLAG_RECOMPUTE)) == 0
    assert lib.moe_check_desc(lib.make_desc(8, 128, 64, 4, 2, "bf16",
                                            lib.MOE_FLAG_ACCUM_DW)) == lib.MOE_EINVAL
    assert lib.moe_check_desc(lib.make_desc(8, 128, 64, 4, 2, "bf16",
                                            lib.MOE_FLAG_ACCUM_DW | lib.MOE_FLAG_DW_FP32)) == 0


def test_sizes_grow_with_the_problem(L):
    small = lib.moe_workspace_size(lib.make_desc(512, 128, 256, 8, 2, "fp32", lib.MOE_FLAG_ROUTER))
    big = lib.moe_workspace_size(lib.make_desc(16384, 2048, 1024, 128, 4, "bf16"))
    assert 0 < small < big
    d = lib.make_desc(16384, 2048, 1024, 128, 4, "bf16")
    s = lib.moe_saved_layout_get(d)
    R = 16384 * 4
    # every saved tensor is 256-byte aligned and the buffers do not overlap
    offs = [s.topk_idx, s.gates, s.counts, s.offsets, s.slot, s.row_token, s.row_gate, s.x_perm,
            s.H13, s.a, s.y_perm]
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
    assert s.y_perm + R * 2048 * 2 <= s.total
    assert s.H13 - s.x_perm >= R * 2048 * 2 and s.a - s.H13 >= R * 2048 * 2


def test_recompute_moves_activations_from_saved_to_workspace(L):
    d = lib.make_desc(16384, 2048, 1024, 128, 4, "bf16")
    r = lib.make_desc(16384, 2048, 1024, 128, 4, "bf16", lib.MOE_FLAG_RECOMPUTE)
    R = 16384 * 4
    acts = R * 2048 * 2 * 2 + R * 1024 * 2 * 3          # x_perm, y_perm, H13, a
    s_d, s_r = lib.moe_saved_layout_get(d), lib.moe_saved_layout_get(r)
    assert s_d.total - s_r.total >= acts
    assert s_r.x_perm == s_r.H13 == s_r.a == s_r.y_perm == s_r.total
    assert s_r.total < 3 * 1024 * 1024                    # routing metadata only
    assert lib.moe_workspace_size(r) - lib.moe_workspace_size(d) >= acts


def test_shared_expert_layout_and_checks(L):
    sh = lib.make_desc(4096, 256, 128, 16, 4, "bf16", lib.MOE_FLAG_SHARED_EXPERT)
    assert lib.moe_check_desc(sh) == 0
    s = lib.moe_saved_layout_get(sh)
    assert s.a_shared - s.H13_shared >= 4096 * 256 * 2 and s.total - s.a_shared >= 4096 * 128 * 2
    plain = lib.moe_saved_layout_get(lib.make_desc(4096, 256, 128, 16, 4, "bf16"))
    assert plain.H13_shared == plain.a_shared == plain.total
    mx = lib.make_desc(4096, 256, 128, 16, 4, "mxfp8", lib.MOE_FLAG_SHARED_EXPERT)
    assert lib.moe_check_desc(mx) == lib.MOE_EUNSUPPORTED


def test_capacity_padded_layout_sizes(L):
    T, d, f, E, k = 4096, 256, 128, 16, 4
    ragged = lib.make_desc(T, d, f, E, k, "bf16")
    padded = lib.make_desc(T, d, f, E, k, "bf16", capacity=1500)
    assert lib.moe_check_desc(padded) == 0
    assert lib.rows_of(padded) == E * 1500 and lib.rows_of(ragged) == T * k
    sp = lib.moe_saved_layout_get(padded)
    assert sp.H13 - sp.x_perm >= E * 1500 * d * 2
    assert lib.moe_workspace_size(padded) > lib.moe_workspace_size(ragged)
    assert lib.moe_check_desc(lib.make_desc(T, d, f, E, k, "bf16", capacity=-1)) == lib.MOE_EINVAL
    assert lib.moe_check_desc(lib.make_desc(T, d, f, E, k, "bf16", capacity=1 << 28)) == \
        lib.MOE_EINVAL


def test_load_stats_struct_layout(L):
    # the C struct: int64 total, four int32, three doubles
    assert lib.LOAD_STATS_BYTES == 48
    assert lib.moe_load_stats_t.mean.offset == 24


def _p(v):
    return ctypes.c_void_p(v)


def test_pointer_and_workspace_errors_before_any_launch(L):
    d = lib.make_desc(64, 128, 64, 8, 2, "bf16")
    ws_need = lib.moe_workspace_size(d)
    good, bad = 0x10000, 0x10008
    args = [_p(good)] * 8
    # null output pointer
    st = L.moe_route(ctypes.byref(d), _p(good), None, *args[2:8], _p(good), ws_need, None)
    assert st == lib.MOE_EINVAL
    # misaligned pointer
    st = L.moe_route(ctypes.byref(d), _p(bad), *args[1:8], _p(good), ws_need, None)
    assert st == lib.MOE_EALIGN
    # workspace too small
    st = L.moe_route(ctypes.byref(d), *args, _p(good), ws_need - 1, None)
    assert st == lib.MOE_EWORKSPACE
    # null workspace
    st = L.moe_dispatch(ctypes.byref(d), _p(good), _p(good), _p(good), None, None, ws_need, None)
    assert st == lib.MOE_EINVAL
    # the MXFP8 scale-factor buffer is reserved
    st = L.moe_dispatch(ctypes.byref(d), _p(good), _p(good), _p(good), _p(good), _p(good),
                        ws_need, None)
    assert st == lib.MOE_EINVAL
    # saved buffer too small for the layer forward
    s = lib.moe_saved_layout_get(d)
    st = L.moe_layer_fwd(ctypes.byref(d), _p(good), _p(good), None, _p(good), _p(good), _p(good),
                         _p(good), s.total - 256, _p(good), ws_need, None)
    assert st == lib.MOE_EWORKSPACE
    # router flag requires Wr
    dr = lib.make_desc(64, 128, 64, 8, 2, "bf16", lib.MOE_FLAG_ROUTER)
    st = L.moe_layer_fwd(ctypes.byref(dr), _p(good), None, None, _p(good), _p(good), _p(good),
                         _p(good), 1 << 40, _p(good), 1 << 40, None)
    assert st == lib.MOE_EINVAL
    assert L.moe_check_desc(None) == lib.MOE_EINVAL


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.status_string(code) not in ("", "unknown status")


def test_binding_refuses_host_and_strided_tensors():
    """The binding passes raw addresses to device kernels: a host tensor or a strided
    view is refused before the library is called."""
    import torch
    with pytest.raises(ValueError, match="device memory"):
        lib._ptr(torch.zeros(4, 4))
    t = torch.zeros(4, 4)
    if torch.cuda.is_available():
        t = t.cuda()
        with pytest.raises(ValueError, match="contiguous"):
            lib._ptr(t.t())
    assert lib._ptr(None) is None and lib._ptr(1234) == 1234


def test_binding_checks_element_types_and_sizes():
    """Each tensor argument is checked against the descriptor (element type, at least
    the elements the call touches) before the library is called."""
    import torch
    T, d, E, k = 8, 128, 4, 2
    desc = lib.make_desc(T, d, 64, E, k, "bf16")
    slot = torch.zeros(T, k, dtype=torch.int32)
    x_perm = torch.zeros(T * k, d, dtype=torch.bfloat16)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="x must be torch.bfloat16"):
        lib.moe_dispatch(desc, torch.zeros(T, d, dtype=torch.float32), slot, x_perm, ws)
    with pytest.raises(ValueError, match="x holds"):
        lib.moe_dispatch(desc, torch.zeros(T - 1, d, dtype=torch.bfloat16), slot, x_perm, ws)
    # (arguments before the one under test are raw addresses, which pass unchecked; the
    # library is never reached because a later argument is refused)
    with pytest.raises(ValueError, match="slot must be torch.int32"):
        lib.moe_dispatch(desc, 0x1000, slot.long(), x_perm, ws)
    with pytest.raises(ValueError, match="x_perm holds"):
        lib.moe_dispatch(desc, 0x1000, 0x2000, x_perm[:-1], ws)
    with pytest.raises(ValueError, match="logits must be torch.float32"):
        lib.moe_router_logits(desc, 0x1000, 0x2000, torch.zeros(T, E, dtype=torch.bfloat16))


def test_product_code_never_reaches_the_oracle():
    """The package (binding, input generators, build) and the CUDA sources share nothing
    with oracle/: no import, include or path to it.  Only tests, the smoke check and the
    bench's CPU-baseline / reference legs may use the oracle."""
    pkg = os.path.join(ROOT, "routing_grouped_gemm_route_b200")
    pat = re.compile(r"(^|\W)(import\s+oracle|from\s+oracle|oracle/|\"oracle|'oracle)")
    bad = []
    for dirpath, _, files in os.walk(pkg):
        for name in files:
            if name.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                path = os.path.join(dirpath, name)
                with open(path, encoding="utf-8") as fh:
                    for i, line in enumerate(fh, 1):
                        if pat.search(line):
                            bad.append(f"{os.path.relpath(path, ROOT)}:{i}")
    for name in os.listdir(os.path.join(ROOT, "include")):
        with open(os.path.join(ROOT, "include", name), encoding="utf-8") as fh:
            if "oracle" in fh.read():
                bad.append(f"include/{name}")
    assert not bad, bad


def test_binding_constants_match_the_header():
    """Every MOE_FLAG_* / MOE_DEV_* / MOE_* status the header defines has the same value in
    the binding (which only passes them through)."""
    import re
    hdr = open(os.path.join(ROOT, "include", "moe.h")).read()
    found = 0
    for name, expr in re.findall(r"#define (MOE_(?:FLAG|DEV)_[A-Z0-9_]+)\s+(\(?[0-9 <]+\)?)", hdr):
        assert getattr(lib, name) == eval(expr), name
        found += 1
    assert found >= 9
    for name, val in re.findall(r"(MOE_E[A-Z]+|MOE_OK)\s*=\s*(-?\d+)", hdr):
        assert getattr(lib, name) == int(val), name
