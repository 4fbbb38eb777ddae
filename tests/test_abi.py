"""The C-ABI library loads, exports every symbol include/vattn.h declares, and
rejects bad arguments synchronously (CPU only: no call here launches work)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "vattn.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(vattn_\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def V():
    import video_dit_local_b200 as V
    return V


def test_every_declared_symbol_is_exported(V):
    names = _declared()
    assert "vattn_sta_fwd" in names and "vattn_dual_bwd" in names
    lib = ctypes.CDLL(V.binding.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # the Python binding offers the same names
    for n in names:
        assert hasattr(V.binding, n), n


def test_library_has_no_libcuda_link_dependency(V):
    import subprocess
    out = subprocess.run(["readelf", "-d", V.binding.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_version(V):
    assert "sm_100a" in V.vattn_version()


def _geom(V, **kw):
    a = dict(batch=1, heads=2, head_dim=64, grid=(4, 8, 8), tile=(2, 4, 4), window=(1, 2, 2), pool=(1, 2, 2))
    a.update(kw)
    return V.make_geom(a["batch"], a["heads"], a["head_dim"], a["grid"], a["tile"], a["window"], a["pool"])


def test_argument_errors(V):
    B = V.binding
    g = _geom(V)
    with pytest.raises(V.VattnError) as e:
        V.vattn_sta_fwd(g, 0, 16, 16, 0.1, 16)
    assert e.value.code == B.VATTN_ERR_INVALID_ARG and "q is NULL" in str(e.value)
    with pytest.raises(V.VattnError) as e:
        V.vattn_sta_fwd(g, 16, 24, 16, 0.1, 16)
    assert e.value.code == B.VATTN_ERR_ALIGN
    with pytest.raises(V.VattnError) as e:
        V.vattn_sta_fwd(_geom(V, grid=(5, 8, 8)), 16, 16, 16, 0.1, 16)
    assert e.value.code == B.VATTN_ERR_SHAPE
    with pytest.raises(V.VattnError) as e:
        V.vattn_sta_fwd(_geom(V, head_dim=96), 16, 16, 16, 0.1, 16)
    assert e.value.code == B.VATTN_ERR_UNSUPPORTED
    with pytest.raises(V.VattnError) as e:
        V.vattn_sta_fwd(_geom(V, tile=(1, 2, 4)), 16, 16, 16, 0.1, 16)   # tile volume 8
    assert e.value.code == B.VATTN_ERR_UNSUPPORTED
    with pytest.raises(V.VattnError) as e:
        V.vattn_pool_kv(_geom(V, pool=(1, 3, 2)), 16, 16, 16, 16)
    assert e.value.code == B.VATTN_ERR_SHAPE
    with pytest.raises(V.VattnError) as e:
        V.vattn_tile_permute(g, 16, 16, 6)
    assert e.value.code == B.VATTN_ERR_INVALID_ARG
    with pytest.raises(V.VattnError) as e:
        V.vattn_dual_fwd(g, 16, 16, 16, 16, 0.1, 16, o_l=16)   # partial set of saved outputs
    assert e.value.code == B.VATTN_ERR_INVALID_ARG
    with pytest.raises(V.VattnError) as e:
        V.vattn_dual_fwd(g, 16, 16, 16, 16, 0.1, 16, workspace=32, ws_bytes=8)
    assert e.value.code == B.VATTN_ERR_WORKSPACE
    with pytest.raises(V.VattnError) as e:
        V.vattn_sta_fwd_host(g, 16, 16, 16, 0.1, 16, 0, 0, 32, 1 << 30)    # chunk of zero slices
    assert e.value.code == B.VATTN_ERR_INVALID_ARG
    with pytest.raises(V.VattnError) as e:
        V.vattn_sta_fwd_host(g, 16, 16, 16, 0.1, 16, 0, 3, 32, 1 << 30)    # more slices than batch*heads
    assert e.value.code == B.VATTN_ERR_INVALID_ARG
    with pytest.raises(V.VattnError) as e:
        V.vattn_sta_fwd_host(g, 16, 16, 16, 0.1, 16, 0, 1, 32, 64)         # two slots needed
    assert e.value.code == B.VATTN_ERR_WORKSPACE
    with pytest.raises(V.VattnError) as e:   # tiles per dim (1, 3, 5) not divisible by h_pool (1, 2, 2)
        V.vattn_hier_fwd(V.make_geom(1, 1, 128, (3, 24, 40), (3, 8, 8), (1, 3, 3), (1, 2, 2)), 16, 16, 16, 0.1, 16,
                         None, 32, 1 << 30)
    assert e.value.code == B.VATTN_ERR_SHAPE and "hierarchical pool" in str(e.value)
    with pytest.raises(V.VattnError) as e:
        V.vattn_hier_fwd(g, 16, 16, 16, 0.1, 16, None, 32, 64)
    assert e.value.code == B.VATTN_ERR_WORKSPACE
    with pytest.raises(V.VattnError) as e:   # t-slice of 6 x 8 = 48 tokens does not divide 128
        V.vattn_sta_fwd_raster(_geom(V, grid=(4, 12, 16), tile=(2, 6, 8)), 16, 16, 16, 0.1, 16)
    assert e.value.code == B.VATTN_ERR_UNSUPPORTED and "t-slice" in str(e.value)
    with pytest.raises(V.VattnError) as e:   # the FP8 forward is d = 128 only
        V.vattn_sta_fwd_fp8(_geom(V, head_dim=64), 16, 16, 16, 0.1, 16, None, 32, 1 << 30)
    assert e.value.code == B.VATTN_ERR_UNSUPPORTED
    with pytest.raises(V.VattnError) as e:
        V.vattn_sta_fwd_fp8(_geom(V, head_dim=128), 16, 16, 16, 0.1, 16, None, 32, 64)
    assert e.value.code == B.VATTN_ERR_WORKSPACE
    with pytest.raises(V.VattnError) as e:
        V.vattn_workspace_size(99, g)
    assert e.value.code == B.VATTN_ERR_INVALID_ARG


def test_empty_batch_is_a_noop(V):
    g = _geom(V, batch=0)
    V.vattn_sta_fwd(g, 0, 0, 0, 0.1, 0)      # nothing to do: no pointer is touched
    V.vattn_dual_fwd(g, 0, 0, 0, 0, 0.1, 0)


def test_workspace_sizes(V):
    g = _geom(V)
    bh, n, npool, d = 2, 256, 64, 64

    def a(x):
        return (x + 255) // 256 * 256
    assert V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD, g) == a(bh * n * d * 2) + 2 * a(bh * npool * d * 2)
    assert V.vattn_workspace_size(V.VATTN_OP_STA_BWD, g) == 2 * a(bh * n * 4)
    # hierarchical forward (pool = h_pool): pooled K, V, then fine O and LSE
    assert V.vattn_workspace_size(V.VATTN_OP_HIER_FWD, g) == (2 * a(bh * npool * d * 2) + a(bh * n * d * 2)
                                                              + a(bh * n * 4))
    # FP8 dual forward: e4m3 Q, K, V, K_p, V_p; two absmax pairs and two single
    # absmax words per batch*head; bf16 O_local, K_p, V_p
    assert V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD_FP8, g) == (
        3 * a(bh * n * d) + 2 * a(bh * npool * d) + 2 * a(bh * 8) + 2 * a(bh * 4) + a(bh * n * d * 2)
        + 2 * a(bh * npool * d * 2))
    # FP8 forward: e4m3 Q, K and V bytes, the (Q, K) absmax pairs, V's absmax
    assert V.vattn_workspace_size(V.VATTN_OP_STA_FWD_FP8, g) == 3 * a(bh * n * d) + a(bh * 8) + a(bh * 4)
    # learned symmetric branch: O_l, Q_p, K_p, V_p, O_p, the upsampled field U (all bf16)
    assert V.vattn_workspace_size(V.VATTN_OP_DUAL_SYM_LEARNED_FWD, g) == (a(bh * n * d * 2) + 4 * a(bh * npool * d * 2)
                                                                       + a(bh * n * d * 2))
    # host-buffer forward, per slot: 8 bf16 token tensors and 2 fp32 rows
    assert V.vattn_workspace_size(V.VATTN_OP_STA_FWD_HOST, g) == 8 * a(bh * n * d * 2) + 2 * a(bh * n * 4)
    assert V.vattn_workspace_size(V.VATTN_OP_DUAL_BWD, g) == (4 * a(bh * n * 4) + 2 * a(bh * npool * d * 4)
                                                              + a(bh * n * d * 4))


def test_kernel_geometry_matches_oracle_inverse_ranges():
    """The device code's window helpers (restated here from the header
    comment: start = clamp(a - w/2, 0, max(n - w, 0))) agree with the oracle."""
    from oracle import vattn_oracle as O
    for n in range(1, 12):
        for w in range(1, 14):
            for a in range(n):
                s = min(max(a - w // 2, 0), max(n - w, 0))
                assert range(s, s + min(w, n)) == O.window_range(a, w, n)


CONSTANTS = ["VATTN_OK", "VATTN_ERR_INVALID_ARG", "VATTN_ERR_SHAPE", "VATTN_ERR_UNSUPPORTED", "VATTN_ERR_ALIGN",
             "VATTN_ERR_CUDA", "VATTN_ERR_DEVICE_TIMEOUT", "VATTN_ERR_WORKSPACE", "VATTN_ERR_DEVICE_BOUNDS",
             "VATTN_OP_DUAL_FWD", "VATTN_OP_STA_BWD", "VATTN_OP_DUAL_BWD", "VATTN_OP_DUAL_SYM_FWD",
             "VATTN_OP_DUAL_SYM_BWD", "VATTN_OP_STA_FWD_HOST", "VATTN_OP_HIER_FWD", "VATTN_OP_HIER_BWD",
             "VATTN_OP_STA_FWD_FP8", "VATTN_OP_DUAL_FWD_FP8", "VATTN_OP_DUAL_SYM_LEARNED_FWD",
             "VATTN_DEBUG_SKIP_ARRIVAL"]


def test_header_is_plain_c_and_links(V, tmp_path):
    """include/vattn.h compiles as C99 (no C++ or torch types in the
    signatures) and a C program links against the library; the constants the
    binding copies from the header agree with it."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_vattn.c"
    src.write_text(
        '#include "vattn.h"\n'
        "#include <stdio.h>\n"
        "int main(void) {\n"
        "  vattn_geom g = {1, 2, 64, 4, 8, 8, {2, 4, 4}, {1, 2, 2}, {1, 1, 1}};\n"
        "  size_t bytes = 0;\n"
        "  int r = vattn_workspace_size(VATTN_OP_DUAL_FWD, &g, &bytes);\n"
        '  printf("%d %zu %s\\n", r, bytes, vattn_version());\n'
        '  printf("%llu\\n", (unsigned long long)VATTN_NOALLOC_SCRATCH_BYTES);\n'
        + "".join(f'  printf("%lld\\n", (long long){c});\n' for c in CONSTANTS)
        + "  return r;\n"
        "}\n")
    exe = tmp_path / "use_vattn"
    lib_dir = os.path.dirname(V.binding.LIB_PATH)
    cmd = [cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", lib_dir, "-l:libvattn.so", f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    lines = out.stdout.strip().split("\n")
    first, second, rest = lines[0], lines[1], lines[2:]
    code, nbytes, version = first.split(maxsplit=2)
    assert code == "0" and int(nbytes) > 0 and "sm_100a" in version
    # the binding's copies of the header's scratch limit, status codes and ops
    assert int(second) == V.binding.VATTN_NOALLOC_SCRATCH_BYTES
    assert len(rest) == len(CONSTANTS)
    for name, value in zip(CONSTANTS, rest):
        assert int(value) == getattr(V.binding, name), name


def test_null_pointers_rejected_before_any_launch(V):
    """Every entry point checks its required pointers on the host."""
    B = V.binding
    g = _geom(V, head_dim=128)
    gp = _geom(V, head_dim=128, pool=(1, 2, 2))
    cases = [
        lambda: V.vattn_sta_fwd_raster(g, 0, 16, 16, 0.1, 16),
        lambda: V.vattn_sta_fwd_fp8(g, 16, 0, 16, 0.1, 16, None, 32, 1 << 30),
        lambda: V.vattn_dual_fwd_fp8(gp, 16, 16, 16, 0, 0.1, 16, 32, 1 << 30),
        lambda: V.vattn_hier_fwd(gp, 16, 16, 0, 0.1, 16, None, 32, 1 << 30),
        lambda: V.vattn_hier_bwd(gp, 16, 16, 16, 16, None, 16, 0.1, 16, 16, 16, 32, 1 << 30),
        lambda: V.vattn_sta_fwd_host(g, 16, 16, 16, 0.1, 0, None, 1, 32, 1 << 30),
    ]
    for f in cases:
        with pytest.raises(V.VattnError) as e:
            f()
        assert e.value.code == B.VATTN_ERR_INVALID_ARG, str(e.value)


def test_misaligned_optional_outputs_rejected(V):
    """Optional outputs (LSE, dg) follow the same 16-byte rule as every other
    pointer, on every entry point that takes one."""
    B = V.binding
    g = _geom(V, head_dim=128)
    cases = [
        lambda: V.vattn_sta_fwd(g, 16, 16, 16, 0.1, 16, lse=20),
        lambda: V.vattn_xwin_fwd(g, 0, 16, 16, 16, 0.1, 16, lse=20),
        lambda: V.vattn_global_fwd(g, 16, 16, 16, 0.1, 16, lse=20),
        lambda: V.vattn_sta_fwd_raster(g, 16, 16, 16, 0.1, 16, lse=20),
        lambda: V.vattn_sta_fwd_fp8(g, 16, 16, 16, 0.1, 16, 20, 32, 1 << 30),
        lambda: V.vattn_hier_fwd(g, 16, 16, 16, 0.1, 16, 20, 32, 1 << 30),
        lambda: V.vattn_dual_fwd(g, 16, 16, 16, 16, 0.1, 16, o_l=16, lse_l=20, o_g=16, lse_g=16, kp=16, vp=16),
        lambda: V.vattn_dual_bwd(g, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, 0.1, 16, 16, 16, 20, 32, 1 << 30),
    ]
    for f in cases:
        with pytest.raises(V.VattnError) as e:
            f()
        assert e.value.code == B.VATTN_ERR_ALIGN and "aligned" in str(e.value), str(e.value)


def test_batch_heads_limit_without_overflow(V):
    """batch*heads >= 2^16 is unsupported, including values whose product
    would overflow 64 bits."""
    B = V.binding
    for batch, heads in [(1, 65536), (256, 256), (1 << 40, 1 << 40)]:
        with pytest.raises(V.VattnError) as e:
            V.vattn_workspace_size(V.VATTN_OP_DUAL_FWD, _geom(V, batch=batch, heads=heads))
        assert e.value.code == B.VATTN_ERR_UNSUPPORTED


def test_shutdown_without_pipeline_is_ok(V):
    """vattn_shutdown with nothing created touches no device and succeeds,
    and may be called repeatedly."""
    V.vattn_shutdown()
    V.vattn_shutdown()
    assert V.vattn_last_error() == ""
