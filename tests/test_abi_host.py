"""Host-side checks of the C ABI: the library loads without a GPU, exports every
call the header declares, validates its arguments before touching CUDA, and
sizes its buffers as documented."""
import ctypes
import os
import re

import pytest

import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")


def _declared_symbols():
    names = set()
    for fn in os.listdir(INCLUDE):
        if fn.endswith(".h"):
            with open(os.path.join(INCLUDE, fn)) as f:
                names |= set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", f.read()))
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(moe.LIB_PATH):
        from mixture_experts_routing_02_b200 import build
        build.build()
    return moe.load_library()


def test_header_declares_the_boundary_calls():
    names = _declared_symbols()
    for required in ("moe_route", "moe_plan_balanced", "moe_dispatch", "moe_expert_ffn", "moe_combine",
                     "moe_layer_fwd"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_symbols()
    assert names, "no MOE_API declarations found"
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(moe.SYMBOLS) <= names | {"moe_status_string"}


def test_every_declared_symbol_has_a_binding_of_the_same_name():
    names = _declared_symbols()
    assert names == set(moe.SYMBOLS)
    for name in names:
        assert callable(getattr(moe, name, None)), f"{name} has no Python binding"


def test_status_strings(lib):
    for code in range(5):
        assert moe.moe_status_string(code).startswith("MOE_")


def _shape(**kw):
    base = dict(T=64, d_model=128, n_experts=8, top_k=2, d_ff=256)
    base.update(kw)
    return moe.shape(**base)


def test_layout_plain_and_capacity(lib):
    assert moe.moe_layout(_shape()) == (8, 128)
    w = syn.SKEWED
    C = 320  # ceil(1.25 * 8192 * 2 / 64)
    s = moe.shape(w.T, w.d, w.E, w.k, w.F, capacity=C)
    assert moe.moe_layout(s) == (64, min(w.T * w.k, C * w.E))
    s = moe.shape(10, 64, 4, 2, 64, capacity=1)
    assert moe.moe_layout(s) == (4, 4)


def test_layout_balanced_plan(lib):
    w = syn.BALANCED
    s = moe.shape(w.T, w.d, w.E, w.k, w.F, n_groups=w.n_groups, replica_slots=w.replica_slots)
    assert moe.moe_layout(s) == (8 * (256 // 8 + 32), w.T * w.k)


def test_dispatch_buffer_matches_moonep_memory_table(lib):
    """MoonEP page, "실제 실험 결과" memory table: the dispatch buffer of one rank
    with S=4096, H=7168, K=8 is 0.44 GiB (S*K rows of H bf16 = 0.4375 GiB)."""
    s = moe.shape(4096, 7168, 256, 8, 2048)
    _, rows = moe.moe_layout(s)
    assert rows * 7168 * 2 == 0.4375 * (1 << 30)
    assert round(rows * 7168 * 2 / (1 << 30), 2) == 0.44


def test_workspace_sizes_grow_with_the_layer(lib):
    small = moe.moe_workspace_size(_shape())
    big = moe.moe_workspace_size(_shape(T=4096))
    assert 0 < small[0] < big[0] and 0 < small[1] < big[1]
    # the layer workspace holds at least Xp, Hp and Yp
    T, d, k, F = 4096, 128, 2, 256
    assert big[1] >= T * k * (2 * d + F) * 2


@pytest.mark.parametrize("kw,code", [
    (dict(T=-1), 1), (dict(top_k=9, n_experts=8), 1), (dict(top_k=0), 1), (dict(n_experts=0), 1),
    (dict(n_groups=3), 1), (dict(n_groups=2, capacity=4), 1), (dict(capacity=-2), 1),
    (dict(n_experts=300, top_k=2), 2), (dict(d_model=100), 2), (dict(d_ff=96), 2),
    (dict(n_experts=16, top_k=9), 2), (dict(T=1 << 29, top_k=2), 2),
    (dict(n_experts=256, n_groups=2, replica_slots=1000, T=64), 2),
    (dict(route_flags=4), 1), (dict(route_flags=-1), 1),
    # expert choice: needs a capacity, no groups, not with softmax-all
    (dict(route_flags=2), 1), (dict(route_flags=3, capacity=8), 1),
    (dict(route_flags=2, capacity=8, n_groups=2), 1),
    (dict(route_flags=2, capacity=1 << 23, T=1 << 23, n_experts=256, top_k=1), 2),
    # re-routing: up to 2^19 (t, j) pairs (each of up to 128 CTAs keeps 4096 in shared memory)
    (dict(route_flags=4, capacity=64, T=1 << 18, top_k=2), 0),
    (dict(route_flags=4, capacity=64, T=(1 << 18) + 1, top_k=2), 2),
])
def test_shape_validation(lib, kw, code):
    s = _shape(**kw)
    n_seg, rows = ctypes.c_int32(), ctypes.c_int32()
    assert lib.moe_layout(ctypes.byref(s), ctypes.byref(n_seg), ctypes.byref(rows)) == code


def test_null_pointers_rejected_before_any_cuda_call(lib):
    s = _shape()
    assert lib.moe_route(ctypes.byref(s), None, None, None, None, None, None, None, None) == 1
    assert lib.moe_combine(ctypes.byref(s), None, None, None, None, None) == 1
    assert lib.moe_expert_ffn(ctypes.byref(s), *([None] * 10)) == 1
    assert lib.moe_plan_balanced(ctypes.byref(s), None, None, None, None, None, None) == 1  # no groups


def test_small_workspace_rejected(lib):
    s = _shape()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    args = [fake] * 9
    rc = lib.moe_dispatch(ctypes.byref(s), fake, fake, 0, *args[:7], fake, fake, 16, None)
    assert rc == 3
    rc = lib.moe_layer_fwd(ctypes.byref(s), fake, fake, None, fake, fake, fake, fake, None, fake, 16, None)
    assert rc == 3


def test_misaligned_workspace_rejected(lib):
    s = _shape()
    fake = ctypes.c_void_p(1 << 20)
    need = moe.moe_workspace_size(s)[1]
    rc = lib.moe_layer_fwd(ctypes.byref(s), fake, fake, None, fake, fake, fake, fake, None,
                           ctypes.c_void_p((1 << 20) + 64), need, None)
    assert rc == 3


def test_expert_choice_layout_and_workspace(lib):
    EC = moe.ROUTE_EXPERT_CHOICE
    assert moe.moe_layout(_shape(route_flags=EC, capacity=10)) == (8, 80)
    assert moe.moe_layout(_shape(route_flags=EC, capacity=1000)) == (8, 8 * 64)   # C' = min(C, T)
    w = syn.EXPERT_CHOICE
    C = -(-w.T * w.k // w.E)
    s = moe.shape(w.T, w.d, w.E, w.k, w.F, capacity=C, route_flags=EC)
    assert moe.moe_layout(s) == (w.E, w.T * w.k)
    disp, layer = moe.moe_workspace_size(s)
    assert disp == 0
    rows = w.T * w.k
    # Xp, Hp, Yp, the [E, T] scores and the [T, E] row map
    assert layer >= rows * (2 * w.d + 2 * w.F + 4 * w.d) + 8 * w.T * w.E


def test_expert_choice_calls_check_the_flag(lib):
    s = _shape()                                     # top-k shape
    ec = _shape(route_flags=moe.ROUTE_EXPERT_CHOICE, capacity=16)
    fake = ctypes.c_void_p(1 << 20)                  # never dereferenced: the flag check comes first
    assert lib.moe_route_scores(ctypes.byref(s), fake, fake, None, fake, None, None) == 1
    assert lib.moe_expert_choose(ctypes.byref(s), *([fake] * 8), None) == 1
    assert lib.moe_combine_expert_choice(ctypes.byref(s), fake, fake, fake, None, fake, None) == 1
    assert lib.moe_dispatch(ctypes.byref(ec), fake, fake, 0, *([fake] * 9), 1 << 30, None) == 1
    assert lib.moe_expert_choose(ctypes.byref(ec), None, *([fake] * 7), None) == 1   # null scores


def test_route_workspace_size(lib):
    """The router's reduction is split only when its ceil(T/128) row tiles leave SMs idle and d
    gives each part at least 4 k-blocks; a split needs S * T * 32*ceil(E/32) fp32 partials."""
    assert moe.moe_route_workspace_size(_shape()) == 0                     # d = 128: too short to split
    w = syn.MIXTRAL_LIKE
    n = moe.moe_route_workspace_size(moe.shape(w.T, w.d, w.E, w.k, w.F))
    assert n >= 2 * w.T * 32 * 4 and n % 256 == 0
    b = syn.BALANCED                                                          # 256 row tiles: no split
    assert moe.moe_route_workspace_size(moe.shape(b.T, b.d, b.E, b.k, b.F, n_groups=b.n_groups,
                                                  replica_slots=b.replica_slots)) == 0


def test_route_ws_checks_before_cuda(lib):
    fake = ctypes.c_void_p(1 << 20)
    ec = _shape(route_flags=moe.ROUTE_EXPERT_CHOICE, capacity=16)
    assert lib.moe_route_ws(ctypes.byref(ec), fake, fake, None, None, fake, fake, None, None, 0, None) == 1
    assert lib.moe_route_scores_ws(ctypes.byref(_shape()), fake, fake, None, fake, None, None, 0, None) == 1
    assert lib.moe_route_ws(ctypes.byref(_shape()), None, fake, None, None, fake, fake, None, None, 0, None) == 1


def test_routing_stats_checks_before_cuda(lib):
    fake = ctypes.c_void_p(1 << 20)                  # never dereferenced: the checks come first
    ec = _shape(route_flags=moe.ROUTE_EXPERT_CHOICE, capacity=16)
    assert lib.moe_routing_stats(ctypes.byref(ec), fake, fake, fake, fake, None) == 1
    s = _shape()
    assert lib.moe_routing_stats(ctypes.byref(s), fake, None, fake, fake, None) == 1
    assert lib.moe_routing_stats(ctypes.byref(s), fake, fake, None, fake, None) == 1
    assert lib.moe_routing_stats(ctypes.byref(s), fake, fake, fake, None, None) == 1


def test_stat_names_follow_the_header():
    """The binding's value names are the header's MOE_STAT_* indices, in order."""
    with open(os.path.join(ROOT, "include", "moe_routing.h")) as f:
        found = dict(re.findall(r"#define MOE_STAT_(\w+) (\d+)", f.read()))
    count = int(found.pop("COUNT"))
    assert count == len(moe.STAT_NAMES)
    assert {n.lower(): int(i) for n, i in found.items()} == {n: i for i, n in enumerate(moe.STAT_NAMES)}


def test_header_is_plain_c_and_the_library_links_from_c(lib, tmp_path):
    """include/moe_routing.h compiles as strict C99, and a C program linked against the library
    calls its host-only entry points (no Python, no torch)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(
        '#include <stdio.h>\n#include "moe_routing.h"\n'
        "int main(void) {\n"
        "    moe_shape_t s = {64, 128, 8, 2, 256, 0, 0, 0, 0, MOE_DTYPE_BF16};\n"
        "    int32_t n_seg = 0, rows = 0;\n"
        "    size_t disp = 0, layer = 0;\n"
        "    if (moe_layout(&s, &n_seg, &rows) != MOE_OK) return 1;\n"
        "    if (moe_workspace_size(&s, &disp, &layer) != MOE_OK) return 2;\n"
        "    s.top_k = 9;\n"
        "    if (moe_layout(&s, &n_seg, &rows) != MOE_ERR_INVALID_ARG) return 3;\n"
        '    printf("%d %d %zu %zu %s\\n", (int)n_seg, (int)rows, disp, layer, moe_status_string(MOE_ERR_WORKSPACE));\n'
        "    return 0;\n}\n")
    pkg = os.path.dirname(moe.LIB_PATH)
    exe = tmp_path / "abi"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", pkg, "-lmoe_b200", "-Wl,-rpath," + pkg], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    disp, layer = moe.moe_workspace_size(_shape())
    assert out[:4] == ["8", "128", str(disp), str(layer)]
    assert out[4] == "MOE_ERR_WORKSPACE:"


def test_missing_library_fails_loudly(tmp_path):
    """No fallback: without the built library every call raises instead of computing elsewhere."""
    with pytest.raises(RuntimeError, match="not built"):
        moe.load_library(str(tmp_path / "libmoe_b200.so"))


def test_out_dtype_is_validated(lib):
    """out_dtype takes MOE_DTYPE_F32 (0) or MOE_DTYPE_BF16 (1); anything else is rejected."""
    for dt, want in ((moe.DTYPE_F32, 0), (moe.DTYPE_BF16, 0), (2, 1), (-1, 1)):
        s = moe.shape(64, 128, 8, 2, 256, out_dtype=dt)
        assert lib.moe_layout(ctypes.byref(s), None, None) == want


def test_ep_sizes_match_moonep_memory_table(lib):
    """MoonEP page, "실제 실험 결과" (memory per rank at S = 4096, H = 7168, K = 8, H' = 2048): the
    dispatch buffer S*K*H*2 bytes = 0.44 GiB and the replica weights of B = 4 slots, B*3*H*H'*2 bytes
    = 0.33 GiB (both printed to two decimals)."""
    R, S, d, E, k, F, B = 8, 4096, 7168, 256, 8, 2048, 4
    s = moe.shape(R * S, d, E, k, F, n_groups=R, replica_slots=B)
    xp_bytes, rep_bytes, n_loc = moe.moe_ep_sizes(s)
    assert xp_bytes == S * k * d * 2 and round(xp_bytes / 2 ** 30, 2) == 0.44
    assert rep_bytes == B * 3 * d * F * 2 and round(rep_bytes / 2 ** 30, 2) == 0.33
    assert n_loc == E // R + B


def test_ep_shapes_are_validated(lib):
    """The moe_ep_* calls need a balanced-plan shape of 1..MOE_EP_MAX_RANKS ranks, without expert
    choice or re-routing."""
    n = ctypes.c_size_t()
    ok = moe.shape(4 * 64, 128, 16, 2, 64, n_groups=4, replica_slots=2)
    assert lib.moe_ep_sizes(ctypes.byref(ok), ctypes.byref(n), None, None) == 0
    no_plan = moe.shape(256, 128, 16, 2, 64)
    assert lib.moe_ep_sizes(ctypes.byref(no_plan), None, None, None) == 1
    too_many = moe.shape(32 * 8, 64, 32, 2, 64, n_groups=32, replica_slots=1)
    assert lib.moe_ep_sizes(ctypes.byref(too_many), None, None, None) == 2
    ec = moe.shape(4 * 64, 128, 16, 2, 64, capacity=8, route_flags=moe.ROUTE_EXPERT_CHOICE)
    assert lib.moe_ep_sizes(ctypes.byref(ec), None, None, None) == 1
    # a rank outside [0, R) is rejected before anything is enqueued
    fake = ctypes.c_void_p(1 << 20)
    assert lib.moe_ep_plan(ctypes.byref(ok), 4, fake, None, fake, fake, fake, None, None) == 1
    assert lib.moe_ep_plan(ctypes.byref(ok), -1, fake, None, fake, fake, fake, None, None) == 1
