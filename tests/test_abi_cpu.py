"""Library loading, exported symbols and host-side validation (no GPU work).

Every call here is rejected by the host-side checks before any CUDA call, or
reads only static data, so it runs on a machine without a GPU.
"""

from __future__ import annotations

import ctypes
import pathlib
import re
import subprocess

import pytest

import exact_io_aware_51_b200 as fa
from exact_io_aware_51_b200 import build as fabuild

ROOT = pathlib.Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "fa.h"


@pytest.fixture(scope="module")
def L():
    fabuild.build()
    return fa.lib()


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_what_the_binding_lists():
    assert declared_functions() == sorted(fa.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", str(fa.lib_path())], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (fa_[a-z0-9_]+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(L, name) is not None


def test_test_only_symbols_live_outside_the_public_header(L):
    """fa_debug_* are declared in csrc/fa_testing.h (not include/fa.h) and exported
    by the library that the binding names for each."""
    testing = ROOT / "exact_io_aware_51_b200" / "csrc" / "fa_testing.h"
    text = re.sub(r"/\*.*?\*/", "", testing.read_text(), flags=re.S)
    declared = sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))
    listed = sorted(n for names in fa.TESTING_EXPORTED.values() for n in names)
    assert declared == listed
    assert not set(declared) & set(declared_functions())
    for lib_name, names in fa.TESTING_EXPORTED.items():
        out = subprocess.run(["nm", "-D", "--defined-only", str(fa.lib_path().parent / lib_name)],
                             capture_output=True, text=True, check=True).stdout
        exported = set(re.findall(r" T (fa_[a-z0-9_]+)$", out, flags=re.M))
        for name in names:
            assert name in exported, (lib_name, name)
    probe = fa.probe_lib()
    assert probe.fa_debug_umma(None, None, None, 64, 64, 0, 0, 0, None) == -1
    # the rate probe validates before touching a device: null buffers, bad shapes, odd pair grids
    assert probe.fa_debug_mma_rate(0, 128, 0, 148, 10, None, None, None, None, None) == -1
    fake = 1 << 20  # never dereferenced: the checks fail first
    assert probe.fa_debug_mma_rate(0, 96, 0, 148, 10, fake, fake, fake, fake, None) == -2
    assert probe.fa_debug_mma_rate(2, 64, 0, 148, 10, fake, fake, fake, fake, None) == -2
    assert probe.fa_debug_mma_rate(2, 128, 0, 147, 10, fake, fake, fake, fake, None) == -2
    assert probe.fa_debug_mma_rate(0, 128, 15, 148, 10, fake, fake, fake, fake, None) == -1
    assert probe.fa_debug_mma_rate(2, 128, 14, 148, 10, fake, fake, fake, fake, None) == -2
    assert probe.fa_debug_mma_rate(0, 256, 13, 148, 10, fake, fake, fake, fake, None) == -2
    assert probe.fa_debug_mma_rate(2, 128, 13, 148, 10, fake, fake, fake, fake, None) == -2


def test_checking_build_exports_the_same_symbols(L):
    """libfa_debug.so (FA_DEBUG: device-side bounds checks) is the product
    library compiled with the checks on: same exported entry points."""
    def exported(path):
        out = subprocess.run(["nm", "-D", "--defined-only", str(path)], capture_output=True, text=True,
                             check=True).stdout
        return set(re.findall(r" T (fa_[a-z0-9_]+)$", out, flags=re.M))
    assert exported(fa.lib_path().parent / "libfa_debug.so") == exported(fa.lib_path())


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -9, -10):
        assert fa.status_string(code) and "unknown" not in fa.status_string(code)
    assert "unknown" in fa.status_string(-99)


def test_validation_rejects_before_touching_the_device(L):
    f = L.fa_fwd
    # null pointers
    assert f(None, None, None, None, None, 1, 1, 128, 64, 0.125, 0, 0, None) == -1
    # unsupported head dim
    assert f(16, 16, 16, 16, 16, 1, 1, 128, 96, 0.125, 0, 0, None) == -2
    # negative sizes, bad dtype, bad scale
    assert f(16, 16, 16, 16, 16, -1, 1, 128, 64, 0.125, 0, 0, None) == -1
    assert f(16, 16, 16, 16, 16, 1, 1, 128, 64, 0.125, 0, 7, None) == -1
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        assert f(16, 16, 16, 16, 16, 1, 1, 128, 64, bad, 0, 0, None) == -1
    # misaligned pointer
    assert f(8, 16, 16, 16, 16, 1, 1, 128, 64, 0.125, 0, 0, None) == -3
    # size limits
    assert f(16, 16, 16, 16, 16, 1, 1, (1 << 22) + 1, 64, 0.125, 0, 0, None) == -8
    assert f(16, 16, 16, 16, 16, 1, 65536, 128, 64, 0.125, 0, 0, None) == -8
    # empty problems are valid no-ops
    assert f(None, None, None, None, None, 0, 4, 128, 64, 0.125, 0, 0, None) == 0
    assert f(None, None, None, None, None, 2, 4, 0, 64, 0.125, 0, 0, None) == 0


def test_backward_validation(L):
    b = L.fa_bwd
    args = [16] * 9
    ws = L.fa_bwd_workspace_size(1, 1, 128, 128, 0)
    # the fp32 backward is not implemented: refused
    assert b(*args, 1, 1, 128, 128, 0.1, 0, 1, 256, ws, None) == -2
    # d = 64 passes the dtype / head-dim check and reaches the alignment check
    bad64 = list(args)
    bad64[3] = 24
    ws64 = L.fa_bwd_workspace_size(1, 1, 128, 64, 0)
    assert b(*bad64, 1, 1, 128, 64, 0.1, 0, 0, 256, ws64, None) == -3
    # workspace missing / too small / misaligned
    assert b(*args, 1, 1, 128, 128, 0.1, 0, 0, None, ws, None) == -4
    assert b(*args, 1, 1, 128, 128, 0.1, 0, 0, 256, ws - 1, None) == -4
    assert b(*args, 1, 1, 128, 128, 0.1, 0, 0, 272, ws, None) == -4
    # misaligned tensor
    bad = list(args)
    bad[7] = 24
    assert b(*bad, 1, 1, 128, 128, 0.1, 0, 0, 256, ws, None) == -3


def test_workspace_is_linear_in_n(L):
    """The method's extra memory is O(N): the fp32 dQ accumulator plus two rows per (b, h),
    and for grids of fewer than three waves of key-tile CTAs, fp32 dK / dV accumulators."""
    def ws(n, H=16, Hkv=None):
        return L.fa_bwd_workspace_size_gqa(2, H, H if Hkv is None else Hkv, n, 128, 0)
    B, H, d = 2, 16, 128
    for n in (4096, 16384):  # 1024 / 4096 CTAs: no split
        expect = B * n * H * d * 4 + 2 * B * H * n * 4
        assert ws(n) == expect
        assert L.fa_bwd_workspace_size(B, H, n, d, 0) == expect
    # B2 H16 N1024: 256 CTAs but only 8 query tiles per key tile, too few to split;
    # B1 H4 N4096: 128 CTAs of 32 query tiles, split (causal / windowed walks)
    assert ws(1024) == B * 1024 * H * d * 4 + 2 * B * H * 1024 * 4
    assert L.fa_bwd_workspace_size(1, 4, 4096, d, 0) == 4096 * 4 * d * 4 * 3 + 2 * 4 * 4096 * 4
    # grouped heads shrink the grid: H64 Hkv8 N4096 is 256 CTAs at B1 (split), 1024 at B4 (7 full
    # waves, no split)
    assert L.fa_bwd_workspace_size_gqa(1, 64, 8, 4096, 128, 0) == \
        4096 * 64 * d * 4 + 2 * 64 * 4096 * 4 + 2 * 4096 * 8 * d * 4
    assert L.fa_bwd_workspace_size_gqa(4, 64, 8, 4096, 128, 0) == 4 * (4096 * 64 * d * 4 + 2 * 64 * 4096 * 4)
    # versus the N x N score matrix standard attention would store (2 bytes each)
    assert ws(16384) < 2 * 16384 * 16384 * H * B
    assert L.fa_bwd_workspace_size(0, 1, 1, 128, 0) == 0
    assert L.fa_bwd_workspace_size(1, 1, 1, 96, 0) == 0
    assert L.fa_bwd_workspace_size_gqa(1, 8, 3, 128, 128, 0) == 0
    # ragged N rounds the per-row arrays up to a multiple of 128 (B4: 2112 CTAs, no split)
    assert L.fa_bwd_workspace_size(4, 16, 4097, 128, 0) == \
        ((4 * 4097 * 16 * 128 * 4 + 255) // 256 * 256) + 2 * ((4 * 16 * 4224 * 4 + 255) // 256 * 256)


def test_python_binding_refuses_cpu_tensors(L):
    import torch
    q = torch.zeros(1, 128, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fwd(q, q, q)


def test_gqa_head_count_validation(L):
    """fa_fwd_gqa / fa_bwd_gqa: Hkv must divide H (grouped-query attention, "Flash Attention"
    (karlkratz.de), "Grouped Query Attention"); checked before any device work."""
    f = L.fa_fwd_gqa
    for H, Hkv in ((8, 3), (8, 0), (8, 16), (8, -1)):
        assert f(16, 16, 16, 16, 16, 1, H, Hkv, 128, 64, 0.125, 0, 0, None) == -1, (H, Hkv)
    # valid groupings get past the head check to the next one (a misaligned pointer)
    for H, Hkv in ((8, 1), (8, 2), (8, 8), (64, 8)):
        assert f(8, 16, 16, 16, 16, 1, H, Hkv, 128, 64, 0.125, 0, 0, None) == -3, (H, Hkv)
    # empty problems stay no-ops
    assert f(None, None, None, None, None, 1, 0, 0, 128, 64, 0.125, 0, 0, None) == 0
    b = L.fa_bwd_gqa
    args = [16] * 9
    ws = L.fa_bwd_workspace_size(1, 8, 128, 128, 0)
    assert b(*args, 1, 8, 3, 128, 128, 0.1, 0, 0, 256, ws, None) == -1
    assert b(*args, 1, 8, 0, 128, 128, 0.1, 0, 0, 256, ws, None) == -1
    bad = list(args)
    bad[7] = 24  # misaligned dK: the head check passed
    assert b(*bad, 1, 8, 2, 128, 128, 0.1, 0, 0, 256, ws, None) == -3


def test_python_binding_checks_gqa_shapes(L):
    import torch
    q = torch.zeros(1, 128, 8, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 128, 3, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="Hkv dividing"):
        fa.fwd(q, k, k)
    k2 = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="Hkv dividing"):
        fa.fwd(q, k2[:, :64], k2[:, :64])
    with pytest.raises(ValueError, match="share one shape"):
        fa.fwd(q, k2, k2[:, :, :1])
    with pytest.raises(ValueError, match="CUDA"):
        fa.fwd(q, k2, k2)  # a valid grouping reaches the device check


def test_window_bound_validation(L):
    """fa_fwd_window / fa_bwd_window: each bound is -1 (open) or >= 0, checked before device work."""
    f = L.fa_fwd_window
    for wl, wr in ((-2, 0), (0, -2), (-5, -5)):
        assert f(16, 16, 16, 16, 16, 1, 2, 2, 128, 64, 0.125, wl, wr, 0, None) == -1, (wl, wr)
    for wl, wr in ((-1, -1), (-1, 0), (0, 0), (4095, 0), (3, 7), (1 << 30, 1 << 30)):
        assert f(8, 16, 16, 16, 16, 1, 2, 2, 128, 64, 0.125, wl, wr, 0, None) == -3, (wl, wr)
    b = L.fa_bwd_window
    args = [16] * 9
    ws = L.fa_bwd_workspace_size(1, 2, 128, 128, 0)
    assert b(*args, 1, 2, 2, 128, 128, 0.1, -2, 0, 0, 256, ws, None) == -1
    bad = list(args)
    bad[7] = 24
    assert b(*bad, 1, 2, 2, 128, 128, 0.1, 64, 0, 0, 256, ws, None) == -3


def test_python_window_bounds():
    assert fa._window_bounds(False, (None, None)) == (-1, -1)
    assert fa._window_bounds(True, (None, None)) == (-1, 0)
    assert fa._window_bounds(True, (4095, None)) == (4095, 0)
    assert fa._window_bounds(True, (10, 5)) == (10, 0)
    assert fa._window_bounds(False, (3, 7)) == (3, 7)
    with pytest.raises(ValueError):
        fa._window_bounds(False, (-1, 0))


def test_fp8_forward_validation(L):
    """fa_fwd_fp8 refuses what it does not implement before touching the device."""
    f = L.fa_fwd_fp8
    ok = (1.0, 1.0, 1.0)
    # d other than 128
    assert f(16, 16, 16, 16, 16, 1, 2, 2, 128, 64, 0.1, *ok, -1, -1, None) == -2
    # bad scales (softmax scale and each tensor scale)
    for bad in ((0.0, 1.0, 1.0, 1.0), (0.1, -1.0, 1.0, 1.0), (0.1, 1.0, float("nan"), 1.0), (0.1, 1.0, 1.0, 0.0)):
        assert f(16, 16, 16, 16, 16, 1, 2, 2, 128, 128, *bad, -1, -1, None) == -1, bad
    # grouping and window checks, then alignment
    assert f(16, 16, 16, 16, 16, 1, 4, 3, 128, 128, 0.1, *ok, -1, -1, None) == -1
    assert f(16, 16, 16, 16, 16, 1, 4, 2, 128, 128, 0.1, *ok, -3, -1, None) == -1
    assert f(8, 16, 16, 16, 16, 1, 4, 2, 128, 128, 0.1, *ok, 64, 0, None) == -3
    assert f(None, None, None, None, None, 0, 4, 2, 128, 128, 0.1, *ok, -1, -1, None) == 0


def test_blocksparse_validation(L):
    """fa_fwd_blocksparse / fa_bwd_blocksparse argument checks (no device work)."""
    f = L.fa_fwd_blocksparse
    # null mask, wrong mask_heads, fp32, too many key blocks
    assert f(16, 16, 16, 16, 16, 1, 4, 4, 256, 128, 0.1, -1, -1, None, 1, 0, None) == -1
    assert f(16, 16, 16, 16, 16, 1, 4, 4, 256, 128, 0.1, -1, -1, 16, 2, 0, None) == -1
    assert f(8, 16, 16, 16, 16, 1, 4, 4, 256, 128, 0.1, -1, -1, 16, 1, 1, None) == -3  # fp32 passes the dtype check
    assert f(16, 16, 16, 16, 16, 1, 4, 4, 4096 * 128 + 1, 128, 0.1, -1, -1, 16, 1, 0, None) == -8
    # valid arguments reach the alignment check
    assert f(8, 16, 16, 16, 16, 1, 4, 4, 256, 128, 0.1, -1, -1, 16, 4, 0, None) == -3
    b = L.fa_bwd_blocksparse
    args = [16] * 9
    ws = L.fa_bwd_workspace_size(1, 4, 256, 128, 0)
    assert b(*args, 1, 4, 4, 256, 128, 0.1, -1, -1, None, 1, 0, 256, ws, None) == -1
    assert b(*args, 1, 4, 4, 256, 128, 0.1, -1, -1, 16, 3, 0, 256, ws, None) == -1


def test_decode_validation(L):
    """fa_decode_paged argument checks, all before any device work."""
    f = L.fa_decode_paged
    # Q, K, V, table, seqlens, O, LSE, B, H, Hkv, d, page_size, num_pages, max_pages, scale, ws, bytes, stream
    ok = dict(B=2, H=8, Hkv=2, d=128, P=16, npg=10, mp=4, sc=0.1)

    def call(ptr=16, q=None, **kw):
        a = {**ok, **kw}
        p = ptr if q is None else q
        return f(p, ptr, ptr, ptr, ptr, ptr, ptr, a["B"], a["H"], a["Hkv"], a["d"], a["P"], a["npg"], a["mp"],
                 a["sc"], None, 0, None)

    assert call(ptr=None) == -1                       # null pointers
    assert call(d=96) == -2                           # head dim
    for p in (0, 4, 12, 48, 8192):                    # page size: a power of two in [8, 4096]
        assert call(P=p) == -2, p
    assert call(Hkv=3) == -1                          # grouping
    assert call(sc=0.0) == -1 and call(sc=float("nan")) == -1
    assert call(npg=0) == -1 and call(mp=0) == -1 and call(B=-1) == -1
    assert call(npg=1 << 28, P=16) == -8              # pool rows beyond 2^31
    assert call(mp=1 << 28, P=16) == -8               # table span beyond 2^31
    assert call(B=65536) == -8
    assert call(q=8) == -3                            # misaligned Q
    assert call(B=0, ptr=None) == 0                   # empty batch
    # workspace sizes: none for a full batch of short sequences, chunks for a long one
    assert L.fa_decode_workspace_size(64, 64, 8, 128, 16, 8) == 0
    n = L.fa_decode_workspace_size(1, 32, 8, 128, 16, 4096)
    assert n > 0 and n % 256 == 0
    assert L.fa_decode_workspace_size(1, 32, 8, 96, 16, 4096) == 0


def test_python_decode_checks_shapes(L):
    import torch
    q = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    k = torch.zeros(4, 16, 2, 128, dtype=torch.bfloat16)
    t = torch.zeros(2, 2, dtype=torch.int32)
    s = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError):
        fa.decode_paged(q, k, k, t, s)                # CPU tensors: no CPU path
    with pytest.raises(ValueError):
        fa.decode_paged(q, k[..., :64], k[..., :64], t, s)
    with pytest.raises(TypeError):
        fa.decode_paged(q, k, k, t.long(), s)


def test_header_is_plain_c_and_links(L, tmp_path):
    """include/fa.h compiles as C99 and a C program linked against libfa.so calls
    the ABI (static-text and host-only entry points; no GPU needed)."""
    src = tmp_path / "use_fa.c"
    src.write_text(
        '#include <stdio.h>\n#include "fa.h"\n'
        "int main(void) {\n"
        "  const char* s = fa_status_string(FA_ERR_WORKSPACE);\n"
        "  size_t ws = fa_bwd_workspace_size(1, 2, 256, 128, FA_BF16);\n"
        "  size_t dws = fa_decode_workspace_size(1, 32, 8, 128, 16, 4096);\n"
        '  printf("%d %s %zu %zu\\n", fa_version(), s, ws, dws);\n'
        "  return (s && ws > 0 && dws > 0) ? 0 : 1;\n"
        "}\n")
    exe = tmp_path / "use_fa"
    lib_dir = fa.lib_path().parent
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", str(HEADER.parent), str(src), "-o", str(exe),
                    "-L", str(lib_dir), "-lfa", f"-Wl,-rpath,{lib_dir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert out[0] == str(L.fa_version())


def test_fp8_blocksparse_validation(L):
    """fa_fwd_fp8_blocksparse: mask_heads must be 1 or H; valid arguments reach the
    alignment check; a null mask is the plain 8-bit forward."""
    f = L.fa_fwd_fp8_blocksparse
    ok = (0.1, 1.0, 1.0, 1.0)
    assert f(16, 16, 16, 16, 16, 1, 4, 2, 256, 128, *ok, -1, -1, 16, 3, None) == -1
    assert f(16, 16, 16, 16, 16, 1, 4, 2, 256, 64, *ok, -1, -1, 16, 1, None) == -2
    assert f(16, 16, 16, 16, 16, 1, 4, 2, 4096 * 128 + 128, 128, *ok, -1, -1, 16, 1, None) == -8
    assert f(8, 16, 16, 16, 16, 1, 4, 2, 256, 128, *ok, -1, -1, 16, 4, None) == -3
    assert f(8, 16, 16, 16, 16, 1, 4, 2, 256, 128, *ok, -1, -1, None, 0, None) == -3
