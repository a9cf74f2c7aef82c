"""The C ABI library on a host without a GPU: it loads, exports every entry point
declared in include/coat.h, and rejects bad arguments with the documented status
codes before making any CUDA call (so these run on CPU)."""
import ctypes
import os
import re

import pytest
import torch

import fp8_optimizer_state_b200 as coat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "coat.h")

OK, INVALID, MISALIGNED, UNSUPPORTED = 0, 1, 2, 3


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(coat_[a-z0-9_]+)\s*\(", src)))


def test_header_and_binding_agree():
    names = declared_functions()
    assert len(names) >= 12
    assert sorted(n for n, _, _ in coat.EXPORTS) == names


def test_binding_argument_counts_match_the_header():
    """Each declaration's parameter count equals the number of argtypes the
    binding gives ctypes (a missing or extra argument would shift every
    later one)."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = dict(re.findall(r"\b(coat_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src))
    exports = {n: args for n, _, args in coat.EXPORTS}
    assert set(decls) == set(exports)
    for name, params in decls.items():
        params = params.strip()
        count = 0 if params in ("", "void") else params.count(",") + 1
        assert count == len(exports[name]), name


def _ctype_of(param):
    """The ctypes type a C parameter declaration must be passed as."""
    param = " ".join(param.split())
    if "*" in param or param.split()[0] in ("cudaStream_t", "coat_multi_plan_t"):
        return "pointer"
    base = param.replace("const ", "").split()[0]
    return {"int64_t": ctypes.c_int64, "int": ctypes.c_int, "coat_fmt": ctypes.c_int,
            "coat_dtype": ctypes.c_int, "float": ctypes.c_float,
            "size_t": ctypes.c_size_t}[base]


def test_binding_argument_types_match_the_header():
    """Each argtype has the C parameter's width and kind: pointers (and the
    stream and plan handles) as pointers, int64_t / int / enum / float /
    size_t as those ctypes types."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = dict(re.findall(r"\b(coat_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src))
    for name, res, args in coat.EXPORTS:
        params = [p for p in decls[name].split(",") if p.strip() not in ("", "void")]
        for i, (param, arg) in enumerate(zip(params, args)):
            want = _ctype_of(param)
            if want == "pointer":
                assert arg is ctypes.c_void_p or hasattr(arg, "_type_") and \
                    issubclass(arg, ctypes._Pointer), (name, i, param)
            else:
                assert arg is want, (name, i, param, arg)


def test_library_exports_every_declared_symbol():
    L = coat.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert coat.coat_version() == 10400


def test_nm_exports_match():
    import shutil
    import subprocess
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("nm not available")
    out = subprocess.run([nm, "-D", "--defined-only", coat.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r" T (coat_[a-z0-9_]+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported


A = 1 << 20   # a fake, 16-byte aligned "device address" (never dereferenced)
HP = dict(lr=1e-3, b1=0.9, b2=0.95, eps=1e-8, wd=0.1, step=1)


def step(ptrs=None, n=1000, group=128, fm=0, fv=0, **kw):
    p = dict(HP)
    p.update(kw)
    ptrs = ptrs or [A] * 9
    return coat.lib().coat_adamw_step(*ptrs, n, group, p["lr"], p["b1"], p["b2"], p["eps"], p["wd"],
                                      p["step"], fm, fv, None)


def test_step_validation():
    assert step(n=-1) == INVALID
    assert step(group=0) == INVALID
    assert step(group=64) == UNSUPPORTED
    assert step(fm=3) == INVALID and step(fv=-1) == INVALID
    assert step(lr=-1.0) == INVALID and step(lr=float("nan")) == INVALID
    assert step(b1=1.0) == INVALID and step(b2=-0.1) == INVALID
    assert step(eps=0.0) == INVALID and step(wd=-0.5) == INVALID
    assert step(step=0) == INVALID
    for i in range(9):
        ptrs = [A] * 9
        ptrs[i] = None
        expect = OK if i == 1 else INVALID     # weight_bf16_out may be NULL
        if expect == INVALID:
            assert step(ptrs) == INVALID, i
        ptrs[i] = A + 8
        assert step(ptrs) == MISALIGNED, i
    # n == 0 is a no-op that needs no pointers and no device
    assert step([None] * 9, n=0) == OK
    assert "aligned" in coat.coat_last_error() or coat.coat_last_error() != ""


def test_wd_scale_validation():
    L = coat.lib()
    one = (ctypes.c_float * 1)(1.0)
    assert L.coat_multi_plan_set_wd_scale(None, ctypes.cast(one, ctypes.c_void_p), None) == INVALID
    assert "plan is NULL" in coat.coat_last_error()


def test_grad_clip_validation():
    """Argument checks of the clipping entry points run before the plan or the
    record is touched (a host buffer stands in for the plan handle)."""
    L = coat.lib()
    fake = ctypes.create_string_buffer(256)
    plan = ctypes.cast(fake, ctypes.c_void_p)
    rec = ctypes.addressof(fake) + 64
    assert L.coat_multi_plan_grad_norm(None, 1.0, rec, None) == INVALID
    assert "plan is NULL" in coat.coat_last_error()
    assert L.coat_multi_plan_grad_norm(plan, 1.0, None, None) == INVALID
    assert "d_clip is NULL" in coat.coat_last_error()
    assert L.coat_multi_plan_grad_norm(plan, 1.0, rec + 4, None) == MISALIGNED
    for bad in (0.0, -1.0, float("nan")):
        assert L.coat_multi_plan_grad_norm(plan, bad, rec, None) == INVALID
        assert "max_norm" in coat.coat_last_error()
    step = lambda **k: L.coat_adamw_step_multi_clipped(
        k.get("plan", plan), k.get("lr", 1e-3), 0.9, 0.95, 1e-8, 0.0, k.get("step", 1),
        k.get("rec", rec), None)
    assert step(plan=None) == INVALID
    assert step(rec=None) == INVALID and "d_clip is NULL" in coat.coat_last_error()
    assert step(rec=rec + 4) == MISALIGNED
    assert step(lr=-1.0) == INVALID
    assert step(step=0) == INVALID
    assert ctypes.sizeof(coat.GradClip) == 24
    # the finalisation after an all-reduce of the ranks' sums of squares
    assert L.coat_grad_clip_finalize(None, 1.0, None) == INVALID
    assert "d_clip is NULL" in coat.coat_last_error()
    assert L.coat_grad_clip_finalize(rec + 4, 1.0, None) == MISALIGNED
    for bad in (0.0, -1.0, float("nan")):
        assert L.coat_grad_clip_finalize(rec, bad, None) == INVALID
        assert "max_norm" in coat.coat_last_error()
    with pytest.raises(ValueError):
        coat.coat_grad_clip_finalize(torch.zeros(16, dtype=torch.uint8), 1.0)


def test_swiglu_validation():
    """Argument checks of the FP8 SwiGLU entry points (fake, never dereferenced
    device addresses)."""
    L = coat.lib()
    ok = lambda **k: coat.Fp8Act(k.get("q", A), k.get("s", A), k.get("k", A), k.get("ldq", 256),
                                 k.get("lds", 2))
    fwd = lambda g=None, u=None, o=None, rows=4, cols=256, fmt=0, ex=0: L.coat_swiglu_fp8_forward(
        ctypes.byref(g or ok()), ctypes.byref(u or ok()), rows, cols, fmt, ex,
        ctypes.byref(o or ok()), None)
    assert fwd(rows=-1) == INVALID
    assert fwd(cols=250) == UNSUPPORTED and "multiple of 16" in coat.coat_last_error()
    assert fwd(fmt=3) == INVALID
    assert fwd(ex=2) == INVALID
    assert fwd(g=ok(q=None)) == INVALID and "gate" in coat.coat_last_error()
    assert fwd(u=ok(q=A + 8)) == MISALIGNED and "up" in coat.coat_last_error()
    assert fwd(o=ok(ldq=264)) == MISALIGNED and "out" in coat.coat_last_error()
    assert fwd(o=ok(s=A + 2)) == MISALIGNED
    assert fwd(g=ok(lds=1)) == INVALID and "strides" in coat.coat_last_error()
    assert fwd(g=ok(ldq=128)) == INVALID
    assert L.coat_swiglu_fp8_forward(None, ctypes.byref(ok()), 4, 256, 0, 0, ctypes.byref(ok()),
                                     None) == INVALID
    assert fwd(rows=0) == OK and fwd(cols=0) == OK
    bwd = lambda d=A, ldd=256, dg=A, ldg=256, du=A, ldu=256, cols=256: \
        L.coat_swiglu_fp8_backward(d, ldd, ctypes.byref(ok()), ctypes.byref(ok()), 4, cols, 0,
                                   dg, ldg, du, ldu, None)
    assert bwd(d=None) == INVALID and "grad_out" in coat.coat_last_error()
    assert bwd(dg=A + 2) == MISALIGNED and "grad_gate" in coat.coat_last_error()
    assert bwd(ldu=260) == MISALIGNED and "grad_up" in coat.coat_last_error()
    assert bwd(ldd=100) == INVALID
    assert bwd(cols=40) == UNSUPPORTED


def test_rmsnorm_validation():
    L = coat.lib()
    act = lambda **k: coat.Fp8Act(k.get("q", A), k.get("s", A), k.get("k", A), k.get("ldq", 4096),
                                  k.get("lds", 32))
    fwd = lambda x=None, o=None, w=A, rows=4, d=4096, eps=1e-6, fmt=0, ex=0: \
        L.coat_rmsnorm_fp8_forward(ctypes.byref(x or act()), w, rows, d, eps, fmt, ex,
                                   ctypes.byref(o or act()), None)
    assert fwd(d=4000) == UNSUPPORTED and "multiple of 128" in coat.coat_last_error()
    assert fwd(d=8192 + 128, x=act(ldq=8320, lds=65), o=act(ldq=8320, lds=65)) == UNSUPPORTED
    assert fwd(eps=0.0) == INVALID and fwd(eps=float("nan")) == INVALID
    assert fwd(w=None) == INVALID and fwd(w=A + 2) == MISALIGNED
    assert fwd(fmt=5) == INVALID and fwd(ex=3) == INVALID and fwd(rows=-1) == INVALID
    assert fwd(x=act(q=A + 4)) == MISALIGNED and fwd(o=act(lds=8)) == INVALID
    assert fwd(rows=0) == OK
    n = ctypes.c_size_t(7)
    assert L.coat_rmsnorm_fp8_workspace_size(4000, ctypes.byref(n)) == UNSUPPORTED and n.value == 0
    assert L.coat_rmsnorm_fp8_workspace_size(4096, None) == INVALID
    bwd = lambda dy=A, dx=A, dw=A, ws=A, wsb=1 << 30, rows=4: L.coat_rmsnorm_fp8_backward(
        dy, 4096, ctypes.byref(act()), A, rows, 4096, 1e-6, 0, dx, 4096, dw, ws, wsb, None)
    assert bwd(dy=None) == INVALID and "dy" in coat.coat_last_error()
    assert bwd(dx=A + 2) == MISALIGNED and bwd(dw=None) == INVALID and bwd(dw=A + 2) == MISALIGNED


def test_header_compiles_as_c99(tmp_path):
    """include/coat.h is a C header: a C99 translation unit that includes it and
    takes the address of every entry point compiles."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if gcc is None or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime_api.h")):
        pytest.skip("gcc or the CUDA headers are not available")
    names = declared_functions()
    src = tmp_path / "use_coat.c"
    src.write_text('#include "coat.h"\n' + "typedef void (*entry)(void);\n" +
                   "entry entry_points[] = {\n" + ",\n".join("  (entry)%s" % n for n in names) +
                   "\n};\nint main(void) { return entry_points[0] == 0; }\n")
    p = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-fsyntax-only",
                        "-I", os.path.join(ROOT, "include"), "-isystem", cuda_inc, str(src)],
                       capture_output=True, text=True)
    assert p.returncode == 0, p.stderr


def test_struct_layouts_match_the_binding(tmp_path):
    """Every struct of include/coat.h has the size and field offsets of the
    binding's ctypes mirror (a C program built against the header prints
    them)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if gcc is None or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime_api.h")):
        pytest.skip("gcc or the CUDA headers are not available")
    mirrors = {"coat_tensor_desc": coat.TensorDesc, "coat_grad_clip": coat.GradClip,
               "coat_fp8_act": coat.Fp8Act, "coat_shard_piece": coat.ShardPiece}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "coat.h"',
             'int main(void) {']
    for cname, py in mirrors.items():
        lines.append('  printf("%s size %%zu\\n", sizeof(%s));' % (cname, cname))
        for field, _ in py._fields_:
            lines.append('  printf("%s %s %%zu\\n", offsetof(%s, %s));'
                         % (cname, field, cname, field))
    lines += ['  return 0;', '}']
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    p = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        "-isystem", cuda_inc, str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert p.returncode == 0, p.stderr
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True,
                               check=True).stdout.splitlines():
        cname, field, value = line.split()
        got[(cname, field)] = int(value)
    for cname, py in mirrors.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for field, _ in py._fields_:
            assert got[(cname, field)] == getattr(py, field).offset, (cname, field)


def test_selftest_budget_validation():
    L = coat.lib()
    assert L.coat_selftest_wait_timeout(999, None) == INVALID
    assert L.coat_selftest_wait_timeout(2000000001, None) == INVALID
    assert "budget_cycles" in coat.coat_last_error()


def test_codec_validation():
    L = coat.lib()
    q = lambda **k: L.coat_group_quantize(k.get("x", A), k.get("xt", 1), k.get("rows", 8),
                                          k.get("cols", 256), k.get("ldx", 256), k.get("gr", 1),
                                          k.get("gc", 128), k.get("expand", 1), k.get("fmt", 0),
                                          k.get("q", A), k.get("ldq", 256), A, A, None)
    assert q(gr=2) == UNSUPPORTED and q(gc=64) == UNSUPPORTED and q(gr=0) == INVALID
    assert q(xt=7) == INVALID and q(fmt=3) == INVALID and q(expand=2) == INVALID
    assert q(rows=-1) == INVALID and q(ldx=100) == INVALID and q(ldq=255) == INVALID
    assert q(x=A + 4) == MISALIGNED and q(q=A + 1) == MISALIGNED
    assert q(ldx=260) == MISALIGNED      # 520-byte bf16 rows
    assert q(ldq=264) == MISALIGNED
    assert q(rows=0) == OK and q(cols=0, x=None) == OK
    d = lambda **k: L.coat_group_dequantize(k.get("q", A), k.get("ldq", 256), A, A, 8, 256,
                                            k.get("gr", 128), 128, k.get("fmt", 1), k.get("out", A),
                                            k.get("ot", 0), k.get("ldo", 256), None)
    assert d(gr=3) == UNSUPPORTED and d(ot=5) == INVALID and d(out=A + 2) == MISALIGNED
    assert L.coat_fp8_encode(A, -1, 0, A, None) == INVALID
    assert L.coat_fp8_encode(A + 2, 10, 0, A, None) == MISALIGNED
    assert L.coat_fp8_encode(A, 10, 9, A, None) == INVALID
    assert L.coat_fp8_decode(A, 0, 0, None, None) == OK


def test_plan_validation():
    L = coat.lib()
    h = ctypes.c_void_p()
    d = coat.TensorDesc(A, None, A, A, A, A, A, A, A, 1000)
    arr = (coat.TensorDesc * 1)(d)
    assert L.coat_multi_plan_create(None, 1, 128, 0, 0, None, ctypes.byref(h)) == INVALID
    assert L.coat_multi_plan_create(ctypes.cast(arr, ctypes.c_void_p), 0, 128, 0, 0, None,
                                    ctypes.byref(h)) == INVALID
    assert L.coat_multi_plan_create(ctypes.cast(arr, ctypes.c_void_p), 1, 256, 0, 0, None,
                                    ctypes.byref(h)) == UNSUPPORTED
    bad = (coat.TensorDesc * 2)(d, coat.TensorDesc(A, None, A + 4, A, A, A, A, A, A, 10))
    assert L.coat_multi_plan_create(ctypes.cast(bad, ctypes.c_void_p), 2, 128, 0, 0, None,
                                    ctypes.byref(h)) == MISALIGNED
    assert "tensor 1" in coat.coat_last_error()
    assert L.coat_adamw_step_multi(None, 1e-3, 0.9, 0.95, 1e-8, 0.1, 1, None) == INVALID
    assert L.coat_multi_plan_destroy(None) == OK
    assert L.coat_multi_plan_info(None, None, None) == INVALID


def test_binding_raises_without_fallback():
    with pytest.raises(coat.CoatError) as ei:
        coat._check(step(group=64))
    assert ei.value.status == UNSUPPORTED


def test_binding_refuses_host_tensors():
    """The binding passes device pointers only: CPU tensors raise before any
    call into the library (there is no CPU path)."""
    import torch
    q = torch.zeros((2, 128), dtype=torch.uint8)
    s = torch.ones((2, 1))
    act = (q, s, s)
    with pytest.raises(ValueError):
        coat.coat_swiglu_fp8_forward(act, act, 0, False, act)
    with pytest.raises(ValueError):
        coat.coat_rmsnorm_fp8_forward(act, torch.ones(128, dtype=torch.bfloat16), 1e-6, 0, False,
                                      act)
    with pytest.raises(ValueError):
        coat.coat_group_quantize(torch.zeros((2, 128), dtype=torch.bfloat16), 1, 128, False, 0,
                                 q, s, s)


def test_binding_shape_checks():
    import torch
    q = torch.zeros((2, 128), dtype=torch.uint8)
    with pytest.raises(ValueError):
        coat._act((q, torch.ones(2), torch.ones(2)))              # 1-D scale
    with pytest.raises(ValueError):
        coat._act((q.t(), torch.ones((128, 1)), torch.ones((128, 1))))   # rows not contiguous
