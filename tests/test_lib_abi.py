"""The C-ABI library loads and exports every entry point declared in include/sparsepr.h, and
its host-side argument checks reject bad configurations before touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

from free_block_sparse_02_b200 import build, configs
from free_block_sparse_02_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "sparsepr.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sparsepr_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version(lib):
    assert lib.sparsepr_version() >= 100
    for code in range(8):
        assert lib.sparsepr_status_string(code)
    assert lib.sparsepr_status_string(0) == b"ok"


def test_workspace_size_for_every_workload(lib):
    for w in configs.WORKLOADS:
        n = _lib.workspace_size(_lib.config_from(w))
        assert n > 0 and n % 256 == 0
    small = _lib.workspace_size(_lib.config_from(configs.workload(0)))
    big = _lib.workspace_size(_lib.config_from(configs.workload(2)))
    assert big > 100 * small


@pytest.mark.parametrize("field,value,code", [
    ("d", 96, 2), ("d", 0, 2), ("N", 0, 1), ("s", 0, 1), ("s", 2000, 1), ("n_kgroups", 0, 1),
    ("n_kgroups", 1025, 1), ("n_kgroups", 2000, 1), ("n_qgroups", 2000, 1), ("P", -1, 1),
    ("P", 5000, 1), ("probe_mode", 7, 1), ("dtype", 3, 1), ("km_iters", 0, 1), ("km_iters_warm", -2, 1),
    ("partition", 2, 1), ("partition", -1, 1), ("repair", 2, 1), ("repair", -1, 1), ("probe_mode", 3, 1),
    ("probe_mode", -1, 1), ("correction", 2, 1), ("correction", -1, 1), ("trunc_rank", -1, 1),
    ("trunc_rank", 65, 1),
])
def test_invalid_configs_are_rejected_on_the_host(lib, field, value, code):
    w = configs.workload(0)
    cfg = _lib.config_from(w, **{field: value})
    n = ctypes.c_size_t(0)
    assert lib.sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == code


@pytest.mark.parametrize("base,over,code", [
    (0, dict(B=0), 1), (0, dict(H=0), 1), (0, dict(n_qgroups=0), 1), (0, dict(fixed_k=-1), 1),
    (1, dict(density=1.5), 1), (1, dict(density=float("nan")), 1), (0, dict(P=2000), 1),
    (0, dict(N=500, n_kgroups=600), 1), (0, dict(N=500, n_qgroups=501), 1),
    (0, dict(lam=float("nan")), 1), (0, dict(lam=float("inf")), 1), (0, dict(km_tol=float("nan")), 1),
    (0, dict(km_iters=10001), 1), (0, dict(km_iters_warm=10001), 1),
    (0, dict(key_rank=-1), 1), (0, dict(key_rank=65), 1),
    # sizes: a call whose element count overflows 64-bit offsets is invalid; one whose row count
    # overflows the kernels' int32 row index is valid but not built
    (0, dict(B=2**31 - 1, H=2**31 - 1, N=2**31 - 1, s=1, n_kgroups=1, n_qgroups=1, P=0), 1),
    (2, dict(H=20000), 2),
])
def test_config_ranges_of_the_header_are_enforced(lib, base, over, code):
    """Every range the header states for a sparsepr_config field is checked on the host, with
    the status code the header gives (INVALID_ARG for a value outside its range, UNSUPPORTED for
    a valid call this build does not run)."""
    cfg = _lib.config_from(configs.workload(base), **over)
    n = ctypes.c_size_t(0)
    assert lib.sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == code


def test_range_edges_are_accepted(lib):
    """The inclusive ends of the ranges pass: s = N, C_k = C_q = N, P = N, density = 1,
    trunc_rank = key_rank = d, and the iteration caps."""
    w = configs.workload(0).replace(N=512)
    for over in (dict(s=512), dict(n_kgroups=512, n_qgroups=512), dict(P=512), dict(density=1.0, fixed_k=0),
                 dict(trunc_rank=64, key_rank=64), dict(km_iters=10000, km_iters_warm=10000)):
        cfg = _lib.config_from(w, **over)
        n = ctypes.c_size_t(0)
        assert lib.sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == 0, over


def test_semantic_partition_without_repair_is_accepted(lib):
    cfg = _lib.config_from(configs.workload(1), partition=configs.PARTITION_SEMANTIC, repair=0)
    n = ctypes.c_size_t(0)
    assert lib.sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == 0 and n.value > 0


def test_random_probes_and_mean_only_correction_are_accepted(lib):
    cfg = _lib.config_from(configs.workload(1), probe_mode=configs.PROBE_RANDOM,
                           correction=configs.CORRECTION_MEAN)
    n = ctypes.c_size_t(0)
    assert lib.sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == 0 and n.value > 0


def test_large_group_counts_are_supported(lib):
    # the pages' own configuration: 1000 key groups, 300 query groups
    cfg = _lib.config_from(configs.workload(2), n_kgroups=1000, n_qgroups=300)
    n = ctypes.c_size_t(0)
    assert lib.sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == 0 and n.value > 0


def test_density_is_checked_only_without_fixed_k(lib):
    n = ctypes.c_size_t(0)
    cfg = _lib.config_from(configs.workload(1), density=0.0)
    assert lib.sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == 1
    cfg = _lib.config_from(configs.workload(0), density=0.0)  # fixed_k > 0
    assert lib.sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == 0


def test_null_and_misaligned_arguments(lib):
    cfg = _lib.config_from(configs.workload(0))
    h = ctypes.c_void_p()
    assert lib.sparsepr_workspace_size(None, None) == 1
    assert lib.sparsepr_plan_create(ctypes.byref(cfg), None, 1 << 30, ctypes.byref(h)) == 4
    assert lib.sparsepr_plan_create(ctypes.byref(cfg), 4096 + 16, 1 << 30, ctypes.byref(h)) == 4
    assert lib.sparsepr_plan_create(ctypes.byref(cfg), 4096, 16, ctypes.byref(h)) == 4
    assert lib.sparsepr_plan(None, None, None, None) == 1
    assert lib.sparsepr_attention(None, None, None, None, None) == 1
    assert lib.sparsepr_fit_apply(None, None, 0, None) == 1
    assert lib.sparsepr_sync(None) == 1
    assert lib.sparsepr_set_wait_limit(None, 0, 100) == 1
    assert lib.sparsepr_set_kmeans_path(None, 0) == 1
    assert lib.sparsepr_set_kernel_events(None, 3, None, None) == 1
    lib.sparsepr_plan_destroy(None)


def test_whole_loop_kmeans_partials_are_carved_only_where_a_side_qualifies(lib):
    """The whole-loop k-means needs per-CTA partial sums in the workspace: a bf16 call with at
    most 128 groups whose points fit in the SMs' shared memory gets them (the mid-size call), a
    call too large to keep its points resident does not (the 13B-DiT layer), and an fp32 call
    never does.  The sizes differ by exactly those buffers when the side's shape changes."""
    def size(w):
        cfg = _lib.config_from(w)
        n = ctypes.c_size_t()
        assert lib.sparsepr_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == 0
        return n.value
    mid = configs.workload(1)
    # the same call with 200 key and query groups does not qualify (more than 128 groups)
    many = mid.replace(n_kgroups=200, n_qgroups=200)
    # extra bytes of the larger group count alone, measured on an fp32 call (never qualifies)
    f32 = mid.replace(dtype=configs.F32)
    grow = size(f32.replace(n_kgroups=200, n_qgroups=200)) - size(f32)
    assert size(many) - size(mid) < grow, "the qualifying call must carry extra partial buffers"
    big = configs.workload(2)
    assert size(big.replace(dtype=configs.F32)) - size(big) == size_difference_of_inputs(big)


def size_difference_of_inputs(w):
    """Workspace bytes that depend on the input dtype alone: the permuted Q, K, V and the probe
    queries, at 4 bytes (fp32) against 2 (bf16) per element."""
    BH = w.B * w.H
    return 2 * (3 * BH * w.N * w.d + BH * max(w.P, 1) * w.d)


def _header_layout(tmp_path, structs, constants):
    """Sizes, field offsets and constant values as a C compiler sees them in include/sparsepr.h:
    a small C program prints them."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "sparsepr.h"', "int main(void) {"]
    for cname, fields in structs.items():
        lines.append(f'  printf("size {cname} %zu\\n", sizeof({cname}));')
        for f in fields:
            lines.append(f'  printf("offset {cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    for c in constants:
        lines.append(f'  printf("const {c} %d\\n", (int){c});')
    lines += ["  return 0;", "}"]
    src, exe = tmp_path / "layout.c", tmp_path / "layout"
    src.write_text("\n".join(lines) + "\n")
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return {k: int(v) for k, v in (line.rsplit(" ", 1) for line in out.splitlines())}


def test_binding_structs_and_constants_match_the_header(tmp_path):
    """The ctypes mirrors of sparsepr_config and sparsepr_head_stats have the header's size and
    field offsets, and the binding's constants equal the header's enumerators, so a change on
    one side that the other misses fails here instead of corrupting calls."""
    mirrors = {"sparsepr_config": _lib.Config, "sparsepr_head_stats": _lib.HeadStats}
    c_field = lambda f: "lambda" if f == "lambda_" else f
    structs = {c: [c_field(f) for f, _ in m._fields_] for c, m in mirrors.items()}
    consts = {
        "SPARSEPR_F32": _lib.SPARSEPR_F32, "SPARSEPR_BF16": _lib.SPARSEPR_BF16,
        "SPARSEPR_PROBE_UNIFORM": configs.PROBE_UNIFORM, "SPARSEPR_PROBE_STRATIFIED": configs.PROBE_STRATIFIED,
        "SPARSEPR_PROBE_RANDOM": configs.PROBE_RANDOM,
        "SPARSEPR_CORRECTION_AFFINE": configs.CORRECTION_AFFINE, "SPARSEPR_CORRECTION_MEAN": configs.CORRECTION_MEAN,
        "SPARSEPR_PARTITION_RESPONSE": configs.PARTITION_RESPONSE,
        "SPARSEPR_PARTITION_SEMANTIC": configs.PARTITION_SEMANTIC,
        "SPARSEPR_KERNEL_BLOCK_SPARSE": _lib.KERNEL_BLOCK_SPARSE,
        "SPARSEPR_KERNEL_KMEANS_ASSIGN": _lib.KERNEL_KMEANS_ASSIGN,
        "SPARSEPR_KERNEL_KMEANS_UPDATE": _lib.KERNEL_KMEANS_UPDATE,
        "SPARSEPR_KERNEL_KMEANS_LOOP": _lib.KERNEL_KMEANS_LOOP,
        "SPARSEPR_OK": 0, "SPARSEPR_ERR_STATE": max(_lib.STATUS),
    }
    consts.update({"SPARSEPR_" + n: getattr(_lib, n) for n in dir(_lib) if n.startswith("Q_")})
    got = _header_layout(tmp_path, structs, consts)
    for cname, m in mirrors.items():
        assert got[f"size {cname}"] == ctypes.sizeof(m), cname
        for f, _ in m._fields_:
            assert got[f"offset {cname}.{c_field(f)}"] == getattr(m, f).offset, (cname, f)
    for c, v in consts.items():
        assert got[f"const {c}"] == v, c
    # every query enumerator of the header has a binding constant
    text = open(os.path.join(ROOT, "include", "sparsepr.h")).read()
    assert set(re.findall(r"\b(SPARSEPR_Q_[A-Z_]+)\s*=", text)) == {c for c in consts if c.startswith("SPARSEPR_Q_")}


def test_static_ridge_fit_rejects_bad_arguments_before_any_device_call(lib):
    """sparsepr_ridge_fit_static checks its arguments first, with the header's codes: null
    pointers, a non-finite lambda, no heads or a negative P are INVALID_ARG; d outside
    {64, 128} is UNSUPPORTED; more than 16 heads or 4096 probe rows exceed its fixed scratch
    (WORKSPACE).  The pointers below are never dereferenced: each case returns before the first
    device call."""
    f = lib.sparsepr_ridge_fit_static
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int32
    f.argtypes = [vp, vp, vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_double, vp, vp, vp]
    fake = 4096
    ok = dict(osp=fake, od=fake, w=fake, heads=2, P=48, d=64, lam=-1.0, A=fake)
    cases = [(dict(A=None), 1), (dict(osp=None), 1), (dict(od=None), 1), (dict(w=None), 1),
             (dict(lam=float("nan")), 1), (dict(lam=float("inf")), 1), (dict(heads=0), 1), (dict(P=-1), 1),
             (dict(d=96), 2), (dict(d=0), 2), (dict(heads=17), 4), (dict(P=4097), 4)]
    for over, code in cases:
        a = dict(ok, **over)
        got = f(a["osp"], a["od"], a["w"], a["heads"], a["P"], a["d"], a["lam"], a["A"], None, None)
        assert got == code, over
