"""Host-side checks of the C-ABI library (no GPU needed).

The shared library must load on a machine without a GPU, export every
function include/fa.h declares, and reject invalid arguments on the host
with a status code and a message, before anything is launched.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fa():
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "_fa_build", os.path.join(ROOT, "exact_attention_149_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import exact_attention_149_b200 as m

    return m


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if fn.endswith(".h"):
            src = open(os.path.join(inc, fn), encoding="utf-8").read()
            names += re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_fwd_kvcache", "fa_fwd_kvcache_int8", "fa_kv_quantize_int8",
              "fa_fwd_kvcache_int4", "fa_kv_quantize_int4",
              "fa_bwd_workspace_size",
              "fa_kvcache_workspace_size", "fa_get_device_status", "fa_last_error", "fa_version"):
        assert n in names


def test_library_exports_every_declared_symbol(fa):
    lib = ctypes.CDLL(fa.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_version(fa):
    assert "sm_100a" in fa.fa_version()


def test_workspace_sizes(fa):
    # -LSE and rowsum(dO * O): two float32 vectors per query head, each row
    # of a sequence in a padded layout of 128 * (T / 128 + B + 1) rows per head
    n = fa.fa_bwd_workspace_size(2, 32, 8192, 128)
    assert n == 2 * 32 * 128 * (16384 // 128 + 2 + 1) * 4
    assert fa.fa_bwd_workspace_size(3, 4, 0, 128, 1000) == 2 * 4 * 128 * (1000 // 128 + 3 + 1) * 4
    # kv-cache: float32 split partials (O and LSE per split and output row),
    # padded to 256 B, then the rotated queries in the 16-bit input type
    assert fa.fa_kvcache_workspace_size(64, 1, 32, 128, 1) == 0
    assert fa.fa_kvcache_workspace_size(64, 1, 32, 128, 16) == 16 * 64 * 32 * 129 * 4
    assert fa.fa_kvcache_workspace_size(3, 5, 7, 64, 2) == (2 * 105 * 65 * 4 + 255) // 256 * 256
    assert fa.fa_kvcache_workspace_size(3, 5, 7, 64, 1, 64) == 105 * 64 * 2
    assert fa.fa_kvcache_workspace_size(3, 5, 7, 64, 2, 32) == 54784 + 105 * 64 * 2


def _fwd_status(fa, **kw):
    args = dict(q=16, k=16, v=16, out=16, lse=16, B=1, Hq=2, Hkv=2, S=128, D=64, scale=0.125,
                causal=0, wl=-1, wr=-1, softcap=0.0, al=None, als=0, cu=None, total=0, dtype=0)
    args.update(kw)
    return fa.lib.fa_fwd(args["q"], args["k"], args["v"], args["out"], args["lse"], args["B"],
                         args["Hq"], args["Hkv"], args["S"], args["D"], args["scale"],
                         args["causal"], args["wl"], args["wr"], args["softcap"], args["al"],
                         args["als"], args["cu"], args["total"], args["dtype"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1),
    (dict(out=None), 1),
    (dict(q=8), 1),                 # misaligned
    (dict(B=0), 1),
    (dict(S=0), 1),
    (dict(Hq=3, Hkv=2), 1),         # Hq not a multiple of Hkv
    (dict(wl=-2), 1),
    (dict(softcap=-1.0), 1),
    (dict(softcap=float("inf")), 1),
    (dict(scale=float("nan")), 1),
    (dict(dtype=7), 1),
    (dict(D=96), 2),                # unsupported head dim
    (dict(D=512), 2),
    (dict(cu=16, total=0), 1),
    (dict(al=18), 1),               # misaligned slopes
    (dict(al=16, als=1), 1),        # batch stride neither 0 nor >= Hq
])
def test_fwd_rejects_bad_arguments(fa, kw, status):
    assert _fwd_status(fa, **kw) == status
    assert fa.fa_last_error() != ""


def test_bwd_rejects_bad_arguments(fa):
    lib = fa.lib
    base = [16] * 9 + [1, 2, 2, 128, 64, 0.125, 0, -1, -1, 0.0, None, 0, None, 0, 0]
    # null dout
    a = list(base)
    a[5] = None
    assert lib.fa_bwd(*a, 16, 1 << 20, None) in (1, 2)
    # workspace too small
    assert lib.fa_bwd(*base, 16, 8, None) in (1, 2)
    # workspace missing
    assert lib.fa_bwd(*base, None, 1 << 20, None) in (1, 2)
    # misaligned ALiBi slopes
    a = list(base)
    a[19] = 18
    assert lib.fa_bwd(*a, 16, 1 << 20, None) == 1


def test_kvcache_rejects_bad_arguments(fa):
    lib = fa.lib

    def call(**kw):
        a = dict(q=16, kn=16, vn=16, kc=16, vc=16, bt=16, cs=16, cos=None, sin=None, out=16,
                 lse=16, B=2, Sq=1, Hq=4, Hkv=2, D=128, ps=256, mp=4, npg=8, rrows=0, rd=0,
                 rint=0, scale=0.1, causal=1, wl=-1, wr=-1, softcap=0.0, al=None, als=0, splits=1,
                 dtype=0, ws=None, wsb=0)
        a.update(kw)
        return lib.fa_fwd_kvcache(a["q"], a["kn"], a["vn"], a["kc"], a["vc"], a["bt"], a["cs"],
                                  a["cos"], a["sin"], a["out"], a["lse"], a["B"], a["Sq"], a["Hq"],
                                  a["Hkv"], a["D"], a["ps"], a["mp"], a["npg"], a["rrows"], a["rd"],
                                  a["rint"], a["scale"], a["causal"], a["wl"], a["wr"],
                                  a["softcap"], a["al"], a["als"], a["splits"], a["dtype"], a["ws"],
                                  a["wsb"], None)

    assert call(kc=None) == 1
    assert call(al=18) == 1                           # misaligned ALiBi slopes
    assert call(bt=None) == 1
    assert call(cs=None) == 1
    assert call(splits=0) == 1
    assert call(ps=100) == 1
    assert call(Hq=3) == 1
    assert call(kn=None) == 1 or call(kn=None) == 3  # k_new without v_new is invalid
    assert call(splits=4, ws=None, wsb=0) == 1        # workspace required
    assert call(D=80) == 2
    assert call(Sq=0) == 1
    rot = dict(cos=16, sin=16, rrows=100, ws=256, wsb=1 << 20)
    assert call(rd=24, **rot) == 1                    # not a multiple of 16
    assert call(rd=256, **rot) == 1                   # wider than D
    assert call(rd=64, **dict(rot, cos=None)) == 1    # table missing
    assert call(rd=64, **dict(rot, rrows=0)) == 1     # empty table
    assert call(rd=64, **dict(rot, sin=18)) == 1      # misaligned table
    assert call(rd=64, **dict(rot, ws=None, wsb=0)) == 1  # rotated queries need a workspace


def test_head_dim_256_forward_and_backward(fa):
    """D = 256 passes the forward's and the backward's host checks (they then
    need a device); D = 512 is rejected by both as unsupported."""
    import torch

    if torch.cuda.is_available():
        # with a device these placeholder pointers would reach a launch; the
        # host checks are what this test covers, the GPU tests run the kernels
        pytest.skip("host-only check")
    want = 3  # FA_ERR_CUDA: every host check passed, no device to run on
    fwd_status = fa.lib.fa_fwd(16, 16, 16, 16, 16, 1, 2, 2, 64, 256, 0.1, 1, -1, -1, 0.0, None, 0,
                               None, 0, 0, None)
    assert fwd_status == want
    a = [16] * 9 + [1, 2, 2, 64, 256, 0.1, 1, -1, -1, 0.0, None, 0, None, 0, 0]
    assert fa.lib.fa_bwd(*a, 256, 1 << 20, None) == want
    a512 = [16] * 9 + [1, 2, 2, 64, 512, 0.1, 1, -1, -1, 0.0, None, 0, None, 0, 0]
    assert fa.lib.fa_bwd(*a512, 256, 1 << 20, None) == 2
    # more query heads than the backward's pre pass takes (8192): unsupported,
    # before the workspace check
    heads = [16] * 9 + [1, 8200, 8200, 64, 128, 0.1, 1, -1, -1, 0.0, None, 0, None, 0, 0]
    assert fa.lib.fa_bwd(*heads, 256, 1 << 20, None) == 2
    heads[10] = heads[11] = 8192
    assert fa.lib.fa_bwd(*heads, 256, 1 << 30, None) == want
    assert fa.lib.fa_fwd(16, 16, 16, 16, 16, 1, 2, 2, 64, 512, 0.1, 1, -1, -1, 0.0, None, 0,
                         None, 0, 0, None) == 2


def test_kvcache_int8_rejects_bad_arguments(fa):
    lib = fa.lib

    def call(**kw):
        a = dict(q=16, kn=16, vn=16, kc=16, vc=16, ks=256, vs=512, bt=16, cs=16, out=16, lse=16,
                 B=2, Sq=1, Hkv=2, ps=256, mp=4, npg=8, ws=None, wsb=0)
        a.update(kw)
        return lib.fa_fwd_kvcache_int8(a["q"], a["kn"], a["vn"], a["kc"], a["vc"], a["ks"], a["vs"],
                                       a["bt"], a["cs"], None, None, a["out"], a["lse"], a["B"],
                                       a["Sq"], 4, a["Hkv"], 128, a["ps"], a["mp"], a["npg"], 0, 0,
                                       0, 0.1, 1, -1, -1, 0.0, None, 0, 1, 0, a["ws"], a["wsb"],
                                       None)

    assert call(ks=None) == 1                          # scales are required
    assert call(vs=None) == 1
    assert call(ks=260) == 1                           # scales 16-byte aligned
    assert call(kc=None) == 1
    assert call(ps=100) == 1
    # a contiguous int8 cache needs a capacity that is a multiple of 64
    assert call(bt=None, mp=1, npg=2, ps=300) == 1

    def quant(**kw):
        a = dict(src=16, codes=16, scales=16, npg=4, ps=64, Hkv=2, D=128, dtype=0)
        a.update(kw)
        return lib.fa_kv_quantize_int8(a["src"], a["codes"], a["scales"], a["npg"], a["ps"], a["Hkv"],
                                       a["D"], a["dtype"], None)

    assert quant(src=None) == 1
    assert quant(src=24) == 1                          # misaligned source
    assert quant(npg=0) == 1
    assert quant(D=96) == 2
    assert quant(dtype=7) == 1


def test_binding_checks_int8_cache_shapes(fa):
    """The binding checks what the C ABI cannot see: the dtype and shape of
    the int8 cache's scale tensors (checked before any device access)."""
    import torch

    q = torch.zeros(2, 1, 4, 128, dtype=torch.bfloat16)
    kc = torch.zeros(3, 64, 2, 128, dtype=torch.int8)
    good = torch.zeros(3, 2, 64)
    cs = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(fa.FaError, match="scales must be float32"):
        fa.fwd_kvcache(q, kc, kc.clone(), cs, None, k_scale=torch.zeros(3, 64, 2), v_scale=good)
    with pytest.raises(fa.FaError, match="take k_scale and v_scale"):
        fa.fwd_kvcache(q, kc, kc.clone(), cs, None, k_scale=good)
    with pytest.raises(fa.FaError, match="take k_scale and v_scale"):
        fa.fwd_kvcache(q, kc, kc.clone(), cs, None)
    with pytest.raises(fa.FaError, match="both be int8"):
        fa.fwd_kvcache(q, kc, kc.to(torch.bfloat16), cs, None, k_scale=good, v_scale=good)
    with pytest.raises(fa.FaError, match="scales must be float32"):
        fa.kv_quantize_int8(torch.zeros(3, 64, 2, 128, dtype=torch.bfloat16), scales=torch.zeros(3, 64, 2))


def test_kvcache_int4_rejects_bad_arguments(fa):
    lib = fa.lib

    def call(**kw):
        a = dict(kc=16, ks=256, vs=512, D=128)
        a.update(kw)
        return lib.fa_fwd_kvcache_int4(16, 16, 16, a["kc"], 16, a["ks"], a["vs"], 16, 16, None, None,
                                       16, 16, 2, 1, 4, 2, a["D"], 256, 4, 8, 0, 0, 0, 0.1, 1, -1,
                                       -1, 0.0, None, 0, 1, 0, None, 0, None)

    assert call(ks=None) == 1
    assert call(kc=None) == 1
    assert call(D=256) == 2         # int4 decode is D = 64 or 128
    assert call(D=96) == 2
    assert lib.fa_kv_quantize_int4(None, 16, 16, 1, 64, 1, 128, 0, None) == 1
    assert lib.fa_kv_quantize_int4(16, 16, 16, 1, 64, 1, 96, 0, None) == 2
    assert lib.fa_kv_quantize_int4(16, 16, 16, 1, 64, 1, 256, 0, None) == 2


def test_valid_call_without_gpu_reports_cuda_error(fa):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd_status(fa) == 3  # FA_ERR_CUDA: no device to launch on
    assert "cuda" in fa.fa_last_error().lower() or "device" in fa.fa_last_error().lower()


def test_missing_library_fails_loudly(tmp_path):
    """The binding raises on import when libfa.so is absent: no fallback."""
    import subprocess
    import sys

    pkg = os.path.join(ROOT, "exact_attention_149_b200")
    dst = tmp_path / "exact_attention_149_b200"
    dst.mkdir()
    (dst / "__init__.py").write_text(open(os.path.join(pkg, "__init__.py"), encoding="utf-8").read())
    r = subprocess.run([sys.executable, "-c", "import exact_attention_149_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libfa.so" in r.stderr
