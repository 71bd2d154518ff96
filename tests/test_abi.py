"""C ABI checks that need no GPU: the library builds for sm_100a and loads,
every entry point declared in include/monarch_attn.h is exported, status
strings exist, and argument validation rejects bad calls before touching
CUDA (so these calls are safe on a machine without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from structured_attention_video_monarch_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "monarch_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(monarch_attn_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def test_header_declares_entry_points():
    names = declared_functions()
    assert "monarch_attn_fwd" in names and "monarch_attn_strerror" in names
    assert len(names) >= 5


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in declared_functions():
        assert name in exported, f"{name} declared but not exported"
        assert hasattr(lib, name)


def test_strerror_and_version(lib):
    for code in range(6):
        s = binding.strerror(code)
        assert isinstance(s, str) and s
    assert binding.strerror(99) == "unknown status"
    assert lib.monarch_attn_version() >= 100
    assert binding.monarch_attn_version() == lib.monarch_attn_version()


def test_binding_has_every_declared_entry_point(lib):
    """The Python binding wraps each C entry point under the header's own name."""
    for name in declared_functions():
        assert callable(getattr(binding, name, None)), f"{name} has no binding wrapper"


def test_bwd_workspace_size_binding_matches_library(lib):
    for args in [(2, 3, 4, 5, 6, 64, 1), (1, 1, 2, 2, 2, 128, 0), (1, 1, 2, 2, 2, 96, 1)]:
        assert binding.monarch_attn_bwd_workspace_size(*args) == lib.monarch_attn_bwd_workspace_size(*args)


def _call(lib, q=16, k=32, v=48, out=4096, B=1, heads=1, T=2, H=4, W=4, d=128, fact=0, th=0, tw=0,
          dtype=1):
    return lib.monarch_attn_fwd(q, k, v, out, B, heads, T, H, W, d, fact, th, tw, dtype, None)


@pytest.mark.parametrize("kwargs", [
    dict(q=0),                      # null pointer
    dict(out=0),
    dict(B=0), dict(heads=0), dict(T=0), dict(H=0), dict(W=-1),
    dict(d=96), dict(d=256),        # unsupported head width
    dict(dtype=3),                  # unknown dtype
    dict(fact=3),                   # unknown factorisation
    dict(fact=1, th=3, tw=2),       # tile does not divide H
    dict(fact=1, th=2, tw=0),
    dict(q=18),                     # misaligned (not 16-byte aligned)
    dict(out=16),                   # out aliases q
])
def test_validation_rejects_without_cuda(lib, kwargs):
    assert _call(lib, **kwargs) == 1  # MONARCH_ERR_INVALID_ARG


def test_unsupported_sizes(lib):
    # disjoint fake addresses far apart; rejected before any CUDA call
    big = 1 << 40
    assert lib.monarch_attn_fwd(16, big, 2 * big, 3 * big, 1, 1, 129, 1, 1, 128, 0, 0, 0, 1, None) == 2
    assert lib.monarch_attn_fwd(16, big, 2 * big, 3 * big, 1, 1, 2, 2, 256, 128, 1, 1, 256, 1,
                                None) == 2


def test_host_entry_rejects_null_host_buffers(lib):
    assert lib.monarch_attn_fwd_host(0, 16, 32, 48, 64, 80, 96, 4096, 1, 1, 2, 4, 4, 128, 0, 0, 0,
                                     1, None) == 1


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.monarch_attn_fwd(x, x, x, 2, 2, 2)


def test_product_package_does_not_import_oracle():
    pkg = os.path.join(ROOT, "structured_attention_video_monarch_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "monarch_oracle" not in text, f


def _strided(lib, sb, sh, sn, B=1, heads=2, T=2, H=4, W=4, d=128, fact=0, th=0, tw=0, dtype=1):
    big = 1 << 40
    return lib.monarch_attn_fwd_strided(16, big, 2 * big, 3 * big, B, heads, T, H, W, d, fact, th, tw,
                                        dtype, sb, sh, sn, None)


def test_strided_validation_without_cuda(lib):
    N, d, heads = 32, 128, 2
    assert _strided(lib, 0, N * d, d) == 1                   # stride below 1
    assert _strided(lib, heads * N * d, N * d, d - 8) == 1   # token rows overlap
    assert _strided(lib, heads * N * d, d, d) == 1           # heads and tokens overlap
    assert _strided(lib, heads * N * d, N * d + 4, d) == 1   # not a 16-byte multiple (bf16)
    # the tiled factorisation and the (f*h, w) split keep the contiguous layout
    assert _strided(lib, N * heads * d, d, heads * d, fact=1, th=2, tw=2) == 2
    assert _strided(lib, N * heads * d, d, heads * d, fact=2) == 2


def test_noalloc_refuses_the_row_split_without_cuda(lib):
    big = 1 << 40
    # the (f*h, w) split needs the library's Y1 scratch: refused before any CUDA call
    assert lib.monarch_attn_fwd_noalloc(16, big, 2 * big, 3 * big, 1, 1, 2, 4, 4, 128, 2, 0, 0, None) == 2


def test_bwd_workspace_size_and_validation_without_cuda(lib):
    size = lib.monarch_attn_bwd_workspace_size
    assert size(1, 2, 3, 4, 5, 64, 0) == 2 * 1 * 2 * 3 * 4 * 5 * 64 * 4
    # bf16 / fp16: 16-bit Y1, O, dY1, fp32 row sums and both stages' LSE, fp32 stage-2 dq/dk parts
    assert size(1, 2, 3, 4, 5, 64, 1) == 2 * 60 * (3 * 64 * 2 + 3 * 4 + 2 * 64 * 4)
    assert size(1, 2, 3, 4, 5, 64, 2) == size(1, 2, 3, 4, 5, 64, 1)
    assert size(1, 2, 3, 4, 5, 64, 3) == 0   # unknown dtype
    assert size(1, 2, 3, 4, 5, 96, 0) == 0   # unsupported head width
    big = 1 << 40
    ptrs = [16 + i * big for i in range(8)]
    ws = 2 * 1 * 1 * 2 * 4 * 4 * 128 * 4

    def call(**kw):
        a = dict(B=1, heads=1, T=2, H=4, W=4, d=128, fact=0, th=0, tw=0, dtype=0, ws=ws, p=ptrs)
        a.update(kw)
        p = a["p"]
        return lib.monarch_attn_bwd(*p, a["ws"], a["B"], a["heads"], a["T"], a["H"], a["W"], a["d"],
                                    a["fact"], a["th"], a["tw"], a["dtype"], None)

    assert call(dtype=1) == 1                     # bf16 needs its larger workspace
    ws16 = size(1, 1, 2, 4, 4, 128, 1)
    assert call(dtype=1, ws=ws16 - 16) == 1
    assert call(dtype=3) == 1                     # unknown dtype
    assert call(dtype=0, fact=2) == 1             # fp32 has no (f*h, w) gradients
    big16 = [16 + i * big for i in range(7)] + [16 + 7 * big]
    assert call(dtype=1, T=129, H=1, W=1, ws=size(1, 1, 129, 1, 1, 128, 1), p=big16) == 2  # T > 128
    assert call(dtype=1, p=ptrs[:4] + [ptrs[1]] + ptrs[5:], ws=ws16) == 1  # dq aliases k
    assert call(ws=ws - 16) == 1                  # workspace too small
    assert call(p=[0] + ptrs[1:]) == 1            # null pointer
    assert call(p=ptrs[:4] + [ptrs[0]] + ptrs[5:]) == 1  # dq aliases q
    assert call(d=96) == 1
    assert call(T=129) == 2
    # a workspace that runs into the buffer before it is refused before any
    # CUDA call (back-to-back buffers that do not overlap are accepted: the
    # GPU tests allocate them that way)
    n = ws // 2
    packed = [16 + i * n for i in range(7)]
    assert call(p=packed + [packed[6] + 16]) == 1


def test_chunk_validation_without_cuda(lib):
    big = 1 << 40
    # q, k, v, k_cache, y1_cache, out, y1_new at disjoint fake addresses
    ptrs = [16 + i * big for i in range(7)]

    def call(p=ptrs, B=1, heads=1, T_old=2, T_new=2, H=4, W=4, d=128, fact=0, th=0, tw=0, dtype=1):
        return lib.monarch_attn_fwd_chunk(*p, B, heads, T_old, T_new, H, W, d, fact, th, tw, dtype, None)

    def swap(i, val):
        p = list(ptrs)
        p[i] = val
        return p

    assert call(T_old=-1) == 1                      # negative context length
    assert call(p=swap(3, 0)) == 1                  # context keys missing
    assert call(p=swap(4, 0)) == 1                  # context stage-1 outputs missing
    assert call(p=swap(5, 0)) == 1                  # no out
    assert call(p=swap(5, ptrs[5] + 8)) == 1        # out misaligned
    assert call(p=swap(3, ptrs[3] + 8)) == 1        # context misaligned
    assert call(p=swap(5, ptrs[6] + 16)) == 1       # out overlaps y1_new
    assert call(p=swap(6, ptrs[4] + 64)) == 1       # y1_new overlaps the context
    assert call(p=swap(5, ptrs[0] + 32)) == 1       # out overlaps q
    assert call(fact=2) == 1                        # the (f*h, w) split has no chunk form
    assert call(dtype=3) == 1
    assert call(T_new=0) == 1
    assert call(T_new=129) == 2                     # stage-1 launch limit


def test_header_is_plain_c(tmp_path):
    # the boundary is a C ABI: the header must compile as strict C99 (and as C++)
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "monarch_attn.h"\nint main(void) { return monarch_attn_version() > 0 ? 0 : 1; }\n')
    inc = os.path.dirname(HEADER)
    for cmd in ([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", "-I", inc, str(src)],
                [gcc, "-x", "c++", "-std=c++11", "-Wall", "-Werror", "-fsyntax-only", "-I", inc, str(src)]):
        out = subprocess.run(cmd, capture_output=True, text=True)
        assert out.returncode == 0, out.stderr


def test_library_links_and_validates_from_c(tmp_path, lib):
    # a plain C program links the library and calls it; only calls that are
    # rejected before any CUDA work (no GPU needed)
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "monarch_attn.h"
int main(void) {
    if (monarch_attn_version() < 100) return 1;
    if (strlen(monarch_attn_strerror(MONARCH_ERR_INVALID_ARG)) == 0) return 2;
    /* null inputs: rejected before anything is queued */
    if (monarch_attn_fwd(NULL, NULL, NULL, NULL, 1, 1, 2, 4, 4, 128, MONARCH_FACT_FRAME, 0, 0,
                         MONARCH_DTYPE_BF16, NULL) != MONARCH_ERR_INVALID_ARG) return 3;
    /* the (f*h, w) split is a valid factorisation value; a bad head width is not supported input */
    if (monarch_attn_fwd((void *)16, (void *)(1ull << 40), (void *)(2ull << 40), (void *)(3ull << 40), 1, 1, 2, 4,
                         4, 96, MONARCH_FACT_ROW, 0, 0, MONARCH_DTYPE_BF16, NULL) != MONARCH_ERR_INVALID_ARG) return 4;
    if (monarch_attn_bwd_workspace_size(1, 2, 3, 4, 5, 64, MONARCH_DTYPE_F32) != (size_t)2 * 2 * 3 * 4 * 5 * 64 * 4)
        return 5;
    printf("ok\n");
    return 0;
}
''')
    exe = tmp_path / "client"
    libdir = os.path.dirname(build.LIB)
    out = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-L", libdir,
                          "-lmonarch_attn", f"-Wl,-rpath,{libdir}", "-o", str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stdout, run.stderr)
