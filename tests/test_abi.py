"""The C-ABI boundary on a machine without a GPU.

Checks that libpdssm.so loads, exports every function include/pdssm.h
declares, that the Python mirror of ``pdssm_problem`` has the C layout, and
that argument errors come back as status codes before anything touches CUDA.
No test here passes a pointer that could reach a kernel launch.
"""
import ctypes
import os
import re
import subprocess

import pytest

import structured_sparse_selective_b200 as pd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pdssm.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pdssm_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert set(_declared_functions()) == set(pd.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(pd.library_path())
    for name in _declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", pd.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert exported == set(_declared_functions()), "only the C ABI may be exported"


def test_problem_struct_layout_matches_c(tmp_path):
    src = tmp_path / "layout.c"
    fields = [f for f, _ in pd.Problem._fields_]
    body = "\n".join(f'  printf("{f} %zu\\n", offsetof(pdssm_problem, {f}));' for f in fields)
    src.write_text(f'#include <stdio.h>\n#include <stddef.h>\n#include "pdssm.h"\nint main(void){{\n'
                   f'{body}\n  printf("sizeof %zu\\n", sizeof(pdssm_problem));\n  return 0;\n}}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                       check=True).stdout.splitlines())
    for f in fields:
        assert int(got[f]) == getattr(pd.Problem, f).offset, f
    assert int(got["sizeof"]) == ctypes.sizeof(pd.Problem)


def test_status_strings():
    for code in range(7):
        assert pd.pdssm_status_string(code).startswith("PDSSM_")
    assert pd.pdssm_status_string(99) == "PDSSM_ERR_UNKNOWN"
    assert re.match(r"^\d+\.\d+\.\d+$", pd.version())


def _pb(**kw):
    base = dict(batch=2, seqlen=100, heads=3, N=16, P=8, K=4, chunk=0, logits_t=pd.F32, in_t=pd.F32,
                d_t=pd.F32, state_t=pd.F32, out_t=pd.F32, flags=0)
    base.update(kw)
    return pd.Problem(**base)


def _ws(pb):
    n = ctypes.c_size_t(0)
    rc = pd._lib.pdssm_workspace_size(ctypes.byref(pb), ctypes.byref(n))
    return rc, n.value


@pytest.mark.parametrize("kw,code", [
    (dict(), OK),
    (dict(N=0), INVALID), (dict(P=0), INVALID), (dict(K=0), INVALID), (dict(batch=-1), INVALID),
    (dict(seqlen=-5), INVALID), (dict(chunk=-1), INVALID), (dict(flags=1 << 7), INVALID),
    (dict(N=129), UNSUPPORTED), (dict(P=129), UNSUPPORTED), (dict(K=65), UNSUPPORTED),
    (dict(N=128, P=128, K=64), OK), (dict(batch=0), OK), (dict(seqlen=0), OK),
    (dict(logits_t=pd.C64), UNSUPPORTED), (dict(in_t=pd.C64), UNSUPPORTED),
    (dict(d_t=pd.C64), UNSUPPORTED), (dict(out_t=pd.C64), UNSUPPORTED), (dict(state_t=pd.BF16), UNSUPPORTED),
    (dict(state_t=pd.C64, d_t=pd.F32, out_t=pd.C64), UNSUPPORTED),
    (dict(state_t=pd.C64, d_t=pd.C64, out_t=pd.F32), UNSUPPORTED),
    (dict(state_t=pd.C64, d_t=pd.C64, out_t=pd.C64, in_t=pd.BF16, logits_t=pd.BF16), OK),
    (dict(d_t=pd.BF16, in_t=pd.BF16, out_t=pd.BF16, logits_t=pd.BF16), OK),
    (dict(heads=70000), UNSUPPORTED),
])
def test_workspace_size_validation(kw, code):
    assert _ws(_pb(**kw))[0] == code


def test_workspace_null_arguments():
    n = ctypes.c_size_t(0)
    assert pd._lib.pdssm_workspace_size(None, ctypes.byref(n)) == INVALID
    pb = _pb()
    assert pd._lib.pdssm_workspace_size(ctypes.byref(pb), None) == INVALID


def test_workspace_is_linear_in_length_and_never_quadratic_in_N():
    """O(L*N) memory (Flash PD-SSM page, Methodology 1): no term grows with N*N."""
    def ws(**kw):
        rc, n = _ws(_pb(**kw))
        assert rc == OK
        return n
    base = dict(batch=4, heads=8, P=32, K=8, chunk=64)
    for N in (16, 32, 64, 128):
        for L in (64, 1000, 18000):
            n = ws(N=N, seqlen=L, **base)
            units = base["batch"] * base["heads"] * L
            # y_loc (P per step) + chunk states (N*P per chunk, T >= P) + pairs + selections + dictionary
            assert n <= units * (2 * N + 2 * base["P"] + 8) * 4 + 8 * 128 * 129 * 4 + 4096, (N, L, n)
    # doubling N at fixed everything else at most doubles the N-dependent part
    a, b = ws(N=64, seqlen=4096, **base), ws(N=128, seqlen=4096, **base)
    assert b < 2.2 * a
    # doubling L doubles it (up to alignment)
    a, b = ws(N=64, seqlen=4096, **base), ws(N=64, seqlen=8192, **base)
    assert abs(b - 2 * a) < 2 * 4096


def test_workspace_follows_the_path():
    """The fused single-kernel path (real state, N = P = 64, bf16 d/B/C/x) needs only the
    error word; the three-kernel path (any other problem, or the reference flag) needs its
    chunk states and local outputs."""
    lm = dict(batch=8, seqlen=2048, heads=32, N=64, P=64, K=16, logits_t=pd.BF16, in_t=pd.BF16,
              d_t=pd.BF16, out_t=pd.BF16)
    rc, fused = _ws(_pb(**lm))
    assert rc == OK and fused == 256
    assert _ws(_pb(**dict(lm, chunk=16))) == (OK, 256)
    assert _ws(_pb(**dict(lm, out_t=pd.F32))) == (OK, 256)
    rc, ref = _ws(_pb(**dict(lm, flags=pd.FLAG_REFERENCE_PATH)))
    assert rc == OK and ref > 100 << 20
    for kw in (dict(chunk=64), dict(K=5), dict(N=32), dict(P=32), dict(d_t=pd.F32), dict(in_t=pd.F32)):
        rc, n = _ws(_pb(**dict(lm, **kw)))
        assert rc == OK and n > 1 << 20, kw


def _call_scan(pb, ws_bytes, **ptrs):
    null = None
    fake = ctypes.c_void_p(4096)  # never reaches a launch: every call below fails validation first
    args = dict(s=fake, idx=fake, d=fake, B=fake, C=fake, x=fake, h0=null, y=fake, h_final=null,
                prod_idx=null, prod_val=null, ws=fake)
    args.update(ptrs)
    return pd._lib.pdssm_scan_fwd(ctypes.byref(pb), args["s"], args["idx"], args["d"], args["B"], args["C"],
                                  args["x"], args["h0"], args["y"], args["h_final"], args["prod_idx"],
                                  args["prod_val"], args["ws"], ws_bytes, None)


@pytest.mark.parametrize("missing", ["s", "idx", "d", "B", "C", "x", "y"])
def test_scan_rejects_null_inputs(missing):
    pb = _pb()
    _, need = _ws(pb)
    assert _call_scan(pb, need, **{missing: None}) == INVALID


def test_scan_rejects_small_or_missing_workspace():
    pb = _pb()
    _, need = _ws(pb)
    assert _call_scan(pb, need - 1) == WORKSPACE
    assert _call_scan(pb, need, ws=None) == WORKSPACE


def test_scan_rejects_misaligned_pointers():
    pb = _pb()
    _, need = _ws(pb)
    assert _call_scan(pb, need, d=ctypes.c_void_p(4098)) == INVALID
    assert _call_scan(pb, need, ws=ctypes.c_void_p(4104)) == INVALID
    assert _call_scan(pb, need, h0=ctypes.c_void_p(4097)) == INVALID


def test_scan_rejects_bad_problem_before_pointers():
    assert _call_scan(_pb(N=200), 1 << 30) == UNSUPPORTED
    assert pd._lib.pdssm_scan_fwd(None, *([None] * 12), 0, None) == INVALID


def test_select_and_forward_validation():
    pb = _pb()
    fake = ctypes.c_void_p(4096)
    assert pd._lib.pdssm_select(ctypes.byref(pb), None, fake, None) == INVALID
    assert pd._lib.pdssm_select(ctypes.byref(pb), fake, None, None) == INVALID
    assert pd._lib.pdssm_select(ctypes.byref(_pb(K=100)), fake, fake, None) == UNSUPPORTED
    _, need = _ws(pb)
    args = [fake] * 6 + [None] * 5 + [fake]  # logits..x, h0/y/h_final/prod_idx/prod_val, s_out
    args[7] = None  # y missing
    assert pd._lib.pdssm_forward(ctypes.byref(pb), *args[:11], None, fake, need, None) == INVALID
    assert pd._lib.pdssm_read_device_check(None, None) == INVALID


def test_binding_refuses_cpu_tensors():
    import torch
    t = torch.zeros(4)
    with pytest.raises(ValueError):
        pd._ptr(t)


def test_default_chunk_keeps_the_workspace_below_the_fixed_chunk_one():
    """The default chunk length (chunk = 0) is never shorter than 64 nor than P, so the
    default workspace never exceeds the one of chunk = max(64, P); on long sequences with
    many (batch, head) slices it picks longer chunks and the workspace shrinks."""
    def ws(**kw):
        rc, n = _ws(_pb(**kw))
        assert rc == OK
        return n
    for kw in (dict(batch=4, heads=8, seqlen=18000, N=32, P=32, K=8),
               dict(batch=16, heads=64, seqlen=8192, N=128, P=64, K=64),
               dict(batch=1, heads=1, seqlen=256, N=8, P=4, K=4),
               dict(batch=8, heads=32, seqlen=2048, N=64, P=128, K=16)):
        fixed = ws(chunk=max(64, kw["P"]), **kw)
        assert ws(chunk=0, **kw) <= fixed, kw
    many = dict(batch=16, heads=64, seqlen=8192, N=128, P=64, K=64)
    assert ws(chunk=0, **many) < ws(chunk=64, **many)


def test_backward_validation():
    """pdssm_bwd_workspace_size serves every shape up to the size limits, and
    pdssm_scan_bwd rejects a non-positive temperature, logits without dlogits (and the
    reverse), missing pointers and a small workspace, before any launch."""
    n = ctypes.c_size_t(0)
    cplx = dict(state_t=pd.C64, d_t=pd.C64, out_t=pd.C64)
    # complex states take twice the checkpoint bytes of real ones; the largest shapes fit
    # (a block's columns are split until its shared memory does), many sequences or few
    for kw in (dict(batch=1024, heads=1), dict(batch=2, heads=3)):
        assert pd._lib.pdssm_bwd_workspace_size(ctypes.byref(_pb(N=128, P=64, K=64, **cplx, **kw)),
                                                ctypes.byref(n)) == OK
        n_c = n.value
        assert pd._lib.pdssm_bwd_workspace_size(ctypes.byref(_pb(N=128, P=64, K=64, **kw)), ctypes.byref(n)) == OK
        assert n_c > 1.9 * n.value
        for c in (cplx, {}):
            assert pd._lib.pdssm_bwd_workspace_size(ctypes.byref(_pb(N=128, P=128, K=64, **c, **kw)),
                                                    ctypes.byref(n)) == OK
    pb = _pb()
    assert pd._lib.pdssm_bwd_workspace_size(ctypes.byref(pb), ctypes.byref(n)) == OK and n.value > 0
    fake = ctypes.c_void_p(4096)

    def call(tau=1.0, logits=fake, dlogits=fake, ws_bytes=None, **drop):
        ptr = dict(s=fake, idx=fake, d=fake, B=fake, C=fake, x=fake, dy=fake, dd=fake, dB=fake, dC=fake, dx=fake)
        for k in drop:
            ptr[k] = None
        return pd._lib.pdssm_scan_bwd(ctypes.byref(pb), logits, ptr["s"], ptr["idx"], ptr["d"], ptr["B"], ptr["C"],
                                      ptr["x"], None, ptr["dy"], None, ctypes.c_float(tau), dlogits, ptr["dd"],
                                      ptr["dB"], ptr["dC"], ptr["dx"], None, fake,
                                      n.value if ws_bytes is None else ws_bytes, None)
    assert call(tau=0.0) == 1 and call(tau=-1.0) == 1 and call(tau=float("inf")) == 1
    assert call(logits=None) == 1 and call(dlogits=None) == 1
    for k in ("s", "idx", "d", "B", "C", "x", "dy", "dd", "dB", "dC", "dx"):
        assert call(**{k: True}) == 1, k
    assert call(ws_bytes=n.value - 1) == 3  # PDSSM_ERR_WORKSPACE


def test_dense_selection_validation():
    """The dictionary hardmax, the fused projection, the soft selection and the scan with
    per-step transitions reject bad sizes, unsupported shapes, missing or misaligned pointers
    and small workspaces with a status, before any launch (fake pointers: nothing is read)."""
    lib, fake, odd = pd._lib, ctypes.c_void_p(4096), ctypes.c_void_p(4098)
    # pdssm_dict_hardmax(K, N, M, idx, stream)
    assert lib.pdssm_dict_hardmax(-1, 8, fake, fake, None) == 1
    assert lib.pdssm_dict_hardmax(4, 0, fake, fake, None) == 1
    assert lib.pdssm_dict_hardmax(4, 129, fake, fake, None) == 2
    assert lib.pdssm_dict_hardmax(0, 8, None, None, None) == OK  # nothing to do
    assert lib.pdssm_dict_hardmax(4, 8, None, fake, None) == 1
    assert lib.pdssm_dict_hardmax(4, 8, odd, fake, None) == 1

    # pdssm_select_proj(pb, D, u, W, s, logits, workspace, bytes, stream)
    def proj(D=128, ws_bytes=256, u=fake, W=fake, s_=fake, logits=None, ws=fake, **kw):
        pb = _pb(**dict(dict(heads=4, K=8), **kw))
        return lib.pdssm_select_proj(ctypes.byref(pb), D, u, W, s_, logits, ws, ws_bytes, None)
    assert proj(D=0) == 1 and proj(heads=0) == 1 and proj(K=0) == 1
    assert proj(K=128) == 2                       # above PDSSM_MAX_K
    assert proj(K=6) == 2                         # not a power of two
    assert proj(D=100) == 2                       # not a multiple of 64
    assert proj(heads=3, K=4) == 2                # heads * K not a multiple of 32
    assert proj(heads=40, K=8) == 2               # 320: above 256 and not a multiple of it
    assert proj(u=None) == 1 and proj(W=None) == 1 and proj(s_=None) == 1
    assert proj(u=odd) == 1 and proj(logits=odd) == 1
    assert proj(ws_bytes=255) == 3 and proj(ws=None) == 3

    # pdssm_soft_select_workspace_size / pdssm_soft_select(pb, logits, M, tau, idx_steps, ws, bytes, stream)
    n = ctypes.c_size_t(0)
    soft = dict(N=64, K=16, logits_t=pd.BF16)
    assert lib.pdssm_soft_select_workspace_size(ctypes.byref(_pb(**soft)), ctypes.byref(n)) == OK
    need = n.value
    assert need >= 256 + 2 * 16 * 64 * 64 * 2  # error word + one dictionary's hi / lo parts
    assert lib.pdssm_soft_select_workspace_size(ctypes.byref(_pb(N=48, K=16)), ctypes.byref(n)) == 2  # N not 2^k
    assert lib.pdssm_soft_select_workspace_size(ctypes.byref(_pb(N=8, K=16)), ctypes.byref(n)) == 2   # N < 16

    def softsel(tau=1.0, logits=fake, M=fake, steps=fake, ws=fake, ws_bytes=None):
        return lib.pdssm_soft_select(ctypes.byref(_pb(**soft)), logits, M, ctypes.c_float(tau), steps, ws,
                                     need if ws_bytes is None else ws_bytes, None)
    assert softsel(tau=0.0) == 1 and softsel(tau=float("nan")) == 1
    assert softsel(logits=None) == 1 and softsel(M=None) == 1 and softsel(steps=None) == 1
    assert softsel(ws_bytes=need - 1) == 3

    # pdssm_scan_fwd_steps: the fused kernel's shape only (N = P = 64, bf16 inputs, real state)
    def steps(idx_steps=fake, **kw):
        pb = _pb(**dict(dict(N=64, P=64, K=16, logits_t=pd.BF16, in_t=pd.BF16, d_t=pd.BF16, out_t=pd.BF16), **kw))
        return lib.pdssm_scan_fwd_steps(ctypes.byref(pb), idx_steps, fake, fake, fake, fake, None, fake, None,
                                        None, None, fake, 256, None)
    assert steps(N=32, P=32) == 2
    assert steps(in_t=pd.F32, d_t=pd.F32) == 2
    assert steps(state_t=pd.C64, d_t=pd.C64, out_t=pd.C64) == 2
    assert steps(idx_steps=None) == 1 and steps(idx_steps=odd) == 1


def test_package_refuses_to_load_without_its_cuda_library(tmp_path):
    """No CPU fallback: a copy of the package without libpdssm.so raises on import."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "structured_sparse_selective_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(os.path.dirname(pd.__file__), "__init__.py"), pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import structured_sparse_selective_b200"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=120,
                       env=dict(os.environ, PYTHONPATH=str(tmp_path)))
    assert r.returncode != 0 and "ImportError" in r.stderr and "libpdssm.so" in r.stderr
