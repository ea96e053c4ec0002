"""The C-ABI library loads, exports every function include/sparse_attn.h declares,
and rejects bad arguments on the host before any launch (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "sparse_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sparse_attn_\w+)\s*\(", src)))


def test_header_and_binding_agree(product):
    assert _declared() == sorted(product.EXPORTS)


def test_library_exports_every_declared_symbol(product):
    lib = ctypes.CDLL(product.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_library_is_sm100a_only(product):
    """The shared library carries sm_100a code (built with -gencode arch=compute_100a,code=sm_100a)."""
    import subprocess
    out = subprocess.run(["cuobjdump", "--list-elf", product.LIB_PATH], capture_output=True,
                         text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    archs = set(re.findall(r"sm_(\d+a?)", out.stdout))
    assert archs == {"100a"}, archs


def _err(product, rc):
    return rc, product._lib.lib().sparse_attn_last_error().decode()


def test_argument_errors_on_host(product):
    L = product._lib.lib()
    pat, _t = product.Pattern(causal=1).to_c()
    h = ctypes.c_void_p()
    # H not a multiple of H_kv
    rc, msg = _err(product, L.sparse_attn_plan_create(ctypes.byref(pat), 1, 6, 4, 128, 128,
                                                      ctypes.byref(h)))
    assert rc == product.SA_ERR_INVALID_ARG and "multiple" in msg
    # unsupported head dim
    rc, msg = _err(product, L.sparse_attn_plan_create(ctypes.byref(pat), 1, 4, 4, 128, 96,
                                                      ctypes.byref(h)))
    assert rc == product.SA_ERR_UNSUPPORTED
    # unsupported block_k
    pat2, _t2 = product.Pattern(causal=1, block_k=32).to_c()
    rc, _ = _err(product, L.sparse_attn_plan_create(ctypes.byref(pat2), 1, 4, 4, 128, 64,
                                                    ctypes.byref(h)))
    assert rc == product.SA_ERR_UNSUPPORTED
    # null tensors to the gather entry
    rc, _ = _err(product, L.sparse_attn_gather(None, None, None, None, None, None, 1, 4, 4, 4,
                                               16, 4, 64, 0.0, None, None))
    assert rc == product.SA_ERR_INVALID_ARG
    # misaligned pointer
    rc, msg = _err(product, L.sparse_attn_gather(8, 16, 16, 16, None, 16, 1, 4, 4, 4, 16, 4, 64,
                                                 0.0, None, None))
    assert rc == product.SA_ERR_INVALID_ARG and "aligned" in msg
    # bad H_idx
    rc, _ = _err(product, L.sparse_attn_gather(16, 16, 16, 16, None, 16, 1, 4, 2, 3, 16, 4, 64,
                                               0.0, None, None))
    assert rc == product.SA_ERR_INVALID_ARG


def test_random_table_out_of_range_is_rejected(product):
    import numpy as np
    tab = np.full((1, 2, 1), 5, np.int32)   # only 2 blocks exist for N=128
    with pytest.raises(product.SparseAttnError) as e:
        product.compile_pattern(product.Pattern(n_random=1, random_block=64, random_table=tab), 1, 128)
    assert e.value.code == product.SA_ERR_INVALID_ARG


def test_no_oracle_in_product_path():
    """The product package never imports, loads or names the oracle."""
    pkg = os.path.join(ROOT, "block_sparse_attention_29_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"\boracle\b|sa_oracle", src), f


def test_struct_layouts_match_the_header(product, tmp_path):
    """The binding's ctypes structs have the header's sizes and field offsets
    (a C program built from include/sparse_attn.h prints them)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {"sa_pattern_t": product._lib.SaPattern, "sa_plan_info_t": product._lib.SaPlanInfo}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "sparse_attn.h"',
             "int main(void) {"]
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'  printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l}
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for f, _ in py._fields_:
            assert got[(cname, f)] == getattr(py, f).offset, (cname, f)


def test_decode_entry_points_reject_bad_arguments_on_host(product):
    """Top-K and window decode: argument errors are found before any launch,
    and the workspace size is the documented layout."""
    L = product._lib.lib()
    S, H, Lk, k = 3, 4, 1001, 50

    def r256(n):
        return (n + 255) // 256 * 256
    Lp = (Lk + 3) // 4 * 4
    want = (r256(S * H * Lp * 4) + r256(S * H * 2048 * 4) + r256(S * H * k * 4) + r256(S * H * 4)
            + r256(S * H * k * 4))
    assert product.decode_topk_workspace_bytes(S, H, Lk, k) == want
    assert product.decode_topk_workspace_bytes(S, H, Lk, 0) == 0

    def topk(**kw):
        a = dict(Q=16, K=16, V=16, lengths=None, O=16, S=S, H=H, Hkv=2, L=Lk, d=128, top_k=k,
                 scale=0.0, idx=None, n=None, lse=None, ws=16, ws_bytes=want)
        a.update(kw)
        return _err(product, L.sparse_attn_decode_topk(
            a["Q"], a["K"], a["V"], a["lengths"], a["O"], a["S"], a["H"], a["Hkv"], a["L"],
            a["d"], a["top_k"], a["scale"], a["idx"], a["n"], a["lse"], a["ws"], a["ws_bytes"],
            None))
    assert topk(top_k=0)[0] == product.SA_ERR_INVALID_ARG
    assert topk(Hkv=3)[0] == product.SA_ERR_INVALID_ARG
    assert topk(d=96)[0] == product.SA_ERR_UNSUPPORTED
    rc, msg = topk(ws_bytes=want - 1)
    assert rc == product.SA_ERR_INVALID_ARG and "workspace" in msg
    rc, msg = topk(ws=24)
    assert rc == product.SA_ERR_INVALID_ARG and "aligned" in msg
    assert topk(O=None)[0] == product.SA_ERR_INVALID_ARG
    # more 8192-key chunks than a grid dimension holds
    big = 65535 * 8192 + 1
    assert topk(L=big, S=1, H=2, ws_bytes=product.decode_topk_workspace_bytes(1, 2, big, k))[0] == \
        product.SA_ERR_UNSUPPORTED

    def window(**kw):
        fields = dict(causal=1, window=64, n_global=2)
        fields.update(kw)
        pat, _t = product.Pattern(**fields).to_c()
        return _err(product, L.sparse_attn_decode_window(16, 16, 16, 16, 16, 2, 4, 2, 128,
                                                         ctypes.byref(pat), None, None))[0]
    assert window(causal=0) == product.SA_ERR_UNSUPPORTED
    assert window(window=0) == product.SA_ERR_UNSUPPORTED
    assert window(dilation=2) == product.SA_ERR_UNSUPPORTED
    assert window(block_local=64) == product.SA_ERR_UNSUPPORTED


def test_plan_refusals_on_host(product):
    """Combinations the kernels do not run are refused when the plan is made,
    before any device allocation."""
    L = product._lib.lib()
    h = ctypes.c_void_p()

    def plan(kernel=product.KERNEL_AUTO, N=600, H=4, Hkv=2, d=128, **fields):
        pat, _t = product.Pattern(**fields).to_c()
        return _err(product, L.sparse_attn_plan_create_ex(ctypes.byref(pat), 1, H, Hkv, N, d,
                                                          kernel, ctypes.byref(h)))[0]
    assert plan(causal=1, window=8, dilation=7) == product.SA_ERR_UNSUPPORTED      # 7 does not divide 600
    assert plan(causal=1, window=8, dilation=3, n_global=2) == product.SA_ERR_UNSUPPORTED
    assert plan(causal=1, window=0, dilation=3) == product.SA_ERR_INVALID_ARG
    assert plan(causal=1, kernel=2) == product.SA_ERR_INVALID_ARG   # no longer a kernel
    assert plan(causal=1, kernel=7) == product.SA_ERR_INVALID_ARG


def test_c_program_uses_the_abi(product, tmp_path):
    """A plain C program built against include/sparse_attn.h and linked to the
    library calls its host-only entry points (pattern compiler, workspace size,
    cache slot, error reporting) with the results the binding gets."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <stdlib.h>
#include "sparse_attn.h"
int main(void) {
    sa_pattern_t p = {0};
    p.causal = 1; p.window = 300; p.n_global = 4; p.block_q = 128; p.block_k = 64;
    int H_pat = 0, T = 0; int64_t n = 0;
    if (sparse_attn_compile_pattern(&p, 2, 1000, 128, 64, &H_pat, &T, &n, NULL, NULL, NULL, NULL))
        return 1;
    int32_t *row = malloc(sizeof(int32_t) * (H_pat * T + 1));
    int32_t *kb = malloc(sizeof(int32_t) * n);
    uint8_t *full = malloc(n);
    int64_t *cnt = malloc(sizeof(int64_t) * n);
    if (sparse_attn_compile_pattern(&p, 2, 1000, 128, 64, &H_pat, &T, &n, row, kb, full, cnt))
        return 2;
    long long pairs = 0, nfull = 0;
    for (int64_t e = 0; e < n; ++e) { pairs += cnt[e]; nfull += full[e]; }
    printf("%d %d %lld %lld %lld\n", H_pat, T, (long long)n, nfull, pairs);
    printf("%zu\n", sparse_attn_decode_topk_workspace(3, 4, 1001, 50));
    printf("%lld\n", (long long)sparse_attn_window_slot(5000, 4096, 4));
    p.dilation = 7;
    int rc = sparse_attn_compile_pattern(&p, 2, 1000, 128, 64, &H_pat, &T, &n, NULL, NULL, NULL, NULL);
    printf("%d %s\n", rc, rc ? "refused" : "accepted");
    printf("%d\n", sparse_attn_last_error()[0] != 0);
    return 0;
}
''')
    exe = tmp_path / "use_abi"
    libdir = os.path.dirname(product.LIB_PATH)
    libname = os.path.basename(product.LIB_PATH)[3:-3]
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, f"-l{libname}", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    row_ptr, kb, full, cnt, H_pat, T = product.compile_pattern(
        product.Pattern(causal=1, window=300, n_global=4), 2, 1000)
    assert out[0].split() == [str(H_pat), str(T), str(len(kb)), str(int(full.sum())),
                              str(int(cnt.sum()))]
    assert int(out[1]) == product.decode_topk_workspace_bytes(3, 4, 1001, 50)
    assert int(out[2]) == product.window_slot(5000, 4096, 4) == 4 + 5000 % 4096
    assert out[3].split() == [str(product.SA_ERR_UNSUPPORTED), "refused"]
    assert out[4] == "1"
