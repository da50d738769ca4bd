"""CPU checks of the C ABI: the library loads, exports every entry point that
include/kda.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def kda():
    import __graft_entry__
    __graft_entry__.build()
    import gated_delta_rule_prologue_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:kda_status|const char \*|size_t|int)\s*(kda_\w+)\s*\(",
                                 text, re.M)))


def test_header_declares_the_hot_path_entry_points():
    names = declared_functions()
    for n in ("kda_prologue", "kda_chunk_fwd", "kda_decode_step", "kda_prologue_chunk_fwd",
              "kda_chunk_fwd_ws", "kda_chunk_fwd_workspace_bytes", "kda_get_device_status",
              "kda_last_error", "kda_version"):
        assert n in names


def test_library_exports_every_declared_symbol(kda):
    out = subprocess.run(["nm", "-D", "--defined-only", kda.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (\w+)$", out, re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(kda.lib, n)


def _exported(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    return {n for n in re.findall(r"\bT (\w+)$", out, re.M) if n.startswith("kda_")}


def test_debug_library_matches_the_release_entry_points(kda):
    """libkda_debug.so (KDA_DEBUG) exports the same C ABI and says which build it is;
    the release build refuses the index-check self-test without touching a device."""
    dbg_path = os.path.join(ROOT, "gated_delta_rule_prologue_b200", "libkda_debug.so")
    assert _exported(dbg_path) == _exported(kda.LIB_PATH)
    dbg = ctypes.CDLL(dbg_path)
    for L in (dbg, kda.lib):
        L.kda_debug_build.restype = ctypes.c_int
        L.kda_debug_build.argtypes = []
    assert dbg.kda_debug_build() == 1
    assert kda.lib.kda_debug_build() == 0
    assert kda.lib.kda_selftest_bounds(4, None) == kda.KDA_ERR_UNSUPPORTED
    assert b"release build" in kda.lib.kda_last_error()


def test_no_oracle_or_fallback_in_product_package():
    pkg = os.path.join(ROOT, "gated_delta_rule_prologue_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in src and "from oracle" not in src, f


def _vp(x):
    return ctypes.c_void_p(x)


ALIGNED = 0x10000          # fake, never dereferenced: validation fails first
MISALIGNED = 0x10008


def test_version_and_last_error(kda):
    assert "sm_100a" in kda.kda_version()
    assert isinstance(kda.lib.kda_last_error(), bytes)


def test_chunk_fwd_rejects_bad_arguments(kda):
    L = kda.lib
    a = _vp(ALIGNED)
    # null q
    st = L.kda_chunk_fwd(None, a, a, a, a, 1.0, None, None, 1, 64, 2, 16, 16, 16, 0, a, None, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"q is NULL" in L.kda_last_error()
    # misaligned k
    st = L.kda_chunk_fwd(a, _vp(MISALIGNED), a, a, a, 1.0, None, None, 1, 64, 2, 16, 16, 16, 0,
                         _vp(ALIGNED * 2), None, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"aligned" in L.kda_last_error()
    # N > 1 without cu_seqlens
    st = L.kda_chunk_fwd(a, a, a, a, a, 1.0, None, None, 3, 64, 2, 16, 16, 16, 0, a, None, None)
    assert st == kda.KDA_ERR_INVALID_ARG
    # unsupported head size / chunk / dtype
    st = L.kda_chunk_fwd(a, a, a, a, a, 1.0, None, None, 1, 64, 2, 48, 48, 16, 0, a, None, None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    st = L.kda_chunk_fwd(a, a, a, a, a, 1.0, None, None, 1, 64, 2, 16, 16, 24, 0, a, None, None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    st = L.kda_chunk_fwd(a, a, a, a, a, 1.0, None, None, 1, 64, 2, 16, 16, 16, 7, a, None, None)
    assert st == kda.KDA_ERR_INVALID_ARG
    # output aliasing an input
    st = L.kda_chunk_fwd(a, _vp(ALIGNED * 4), _vp(ALIGNED * 8), _vp(ALIGNED * 12),
                         _vp(ALIGNED * 16), 1.0, None, None, 1, 64, 2, 16, 16, 16, 0, a, None,
                         None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"overlaps" in L.kda_last_error()
    # negative sizes
    st = L.kda_chunk_fwd(a, a, a, a, a, 1.0, None, None, 1, -1, 2, 16, 16, 16, 0, a, None, None)
    assert st == kda.KDA_ERR_INVALID_ARG


def test_prologue_and_decode_reject_bad_arguments(kda):
    L = kda.lib
    a = _vp(ALIGNED)
    st = L.kda_prologue(None, a, None, None, None, 1, 8, 2, 16, 1, 1, _vp(2 * ALIGNED),
                        _vp(3 * ALIGNED), _vp(4 * ALIGNED), None)
    assert st == kda.KDA_ERR_INVALID_ARG
    st = L.kda_prologue(a, a, None, None, None, 1, 8, 2, 24, 1, 1, _vp(2 * ALIGNED),
                        _vp(3 * ALIGNED), _vp(4 * ALIGNED), None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    st = L.kda_prologue(a, a, _vp(5 * ALIGNED), _vp(5 * ALIGNED), None, 1, 8, 2, 16, 1, 0,
                        _vp(2 * ALIGNED), _vp(3 * ALIGNED), _vp(4 * ALIGNED), None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"cache_out overlaps" in L.kda_last_error()
    st = L.kda_decode_step(a, a, a, a, a, 1.0, None, 4, 2, 16, 1, _vp(2 * ALIGNED), None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"state is NULL" in L.kda_last_error()
    st = L.kda_decode_step(a, a, a, a, a, 1.0, a, 4, 2, 100, 1, _vp(2 * ALIGNED), None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    st = L.kda_get_device_status(None)
    assert st == kda.KDA_ERR_INVALID_ARG


def test_fused_prefill_rejects_bad_arguments(kda):
    L = kda.lib
    a = _vp(ALIGNED)
    # D != 128 is outside the fused path's domain
    st = L.kda_prologue_chunk_fwd(a, a, None, None, a, a, 1.0, None, None, 1, 8, 2, 64, 1,
                                  _vp(2 * ALIGNED), None, None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    # float32 projections are not supported by the fused path
    st = L.kda_prologue_chunk_fwd(a, a, None, None, a, a, 1.0, None, None, 1, 8, 2, 128, 0,
                                  _vp(2 * ALIGNED), None, None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    # missing g
    st = L.kda_prologue_chunk_fwd(a, a, None, None, None, a, 1.0, None, None, 1, 8, 2, 128, 1,
                                  _vp(2 * ALIGNED), None, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"g is NULL" in L.kda_last_error()
    # o aliasing x
    st = L.kda_prologue_chunk_fwd(a, _vp(8 * ALIGNED), None, None, _vp(4 * ALIGNED),
                                  _vp(6 * ALIGNED), 1.0, None, None, 1, 8, 2, 128, 1, a, None,
                                  None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"overlaps" in L.kda_last_error()


def test_chunk_workspace_size(kda):
    """Two-pass scratch: a 1 KiB-aligned int32 chunk index and segment index of
    N + 1 entries each, then one record per (chunk, head) for ceil(T/64) + N
    chunks per head, then (segment length L > 0) three 64 KiB fp32 blocks per
    (segment, head) for at most N + floor((T + 63 N) / 64 / L) segments;
    nothing for calls that do not take the tensor-core path."""
    import torch
    f = kda.kda_chunk_fwd_workspace_bytes
    fs = kda.kda_chunk_fwd_segmented_workspace_bytes
    rec = fs(1, 64, 1, 128, 128, 64, torch.bfloat16, 0) - 1024
    assert rec > 0 and rec % 32 == 0   # two records (ceil(64/64) + N = 2), 16-byte multiples
    rec //= 2
    for N, T, H in ((1, 32768, 96), (16, 93891, 32), (300, 1000, 2), (1, 4096, 8), (3, 999, 2)):
        header = ((N + 1) * 8 + 1023) // 1024 * 1024
        base = header + ((T + 63) // 64 + N) * H * rec
        for L in (0, 1, 3, 10):
            seg = 0 if L == 0 else (N + (T + 63 * N) // 64 // L) * H * 3 * 65536
            assert fs(N, T, H, 128, 128, 64, torch.float16, L) == base + seg
        L = kda.kda_chunk_fwd_segment_chunks(N, T, H)
        assert f(N, T, H, 128, 128, 64, torch.float16) == fs(N, T, H, 128, 128, 64,
                                                             torch.float16, L)
    assert f(1, 64, 1, 128, 128, 64, torch.float32) == 0
    assert f(1, 64, 1, 64, 64, 64, torch.bfloat16) == 0
    assert f(1, 64, 1, 128, 128, 32, torch.bfloat16) == 0
    assert f(1, 0, 1, 128, 128, 64, torch.bfloat16) == 0
    assert fs(1, 64, 1, 128, 128, 64, torch.bfloat16, -1) == 0


def test_segment_length_choice(kda):
    """Sequences are split only when the (sequence, head, 32-value-channel)
    chains fill fewer than two CTAs per SM of 148, and only into three or more
    segments (with two, the transition and output passes walk as many chunks
    one after the other as the whole sequence does)."""
    sc = kda.kda_chunk_fwd_segment_chunks
    assert sc(1, 32768, 96) == 0        # 384 chains: whole sequences
    assert sc(16, 130000, 32) == 0      # varlen batch of 16 x 32 heads
    assert sc(1, 4096, 32) == 0         # 128 chains of 64 chunks: no split pays
    assert sc(1, 4096, 8) == 8          # 64 chunks, 8 heads: 8 segments of 8
    assert sc(1, 256, 2) == 0           # 4 chunks
    assert sc(2, 64, 1) == 0
    assert sc(0, 64, 1) == 0 and sc(1, -1, 1) == 0 and sc(1, 64, 0) == 0
    for T, H in ((1000, 2), (8192, 2), (16384, 8), (32768, 16), (131072, 1), (4096, 16)):
        L = sc(1, T, H)
        nch = (T + 63) // 64
        assert L > 0 and (nch + L - 1) // L >= 3, (T, H, L)


def test_chunk_fwd_segmented_rejects_bad_arguments(kda):
    """Argument checks run before any device call: a negative segment length,
    a NULL or short workspace, and sizes off the tensor-core path."""
    import torch
    L = kda.lib
    T, H = 640, 2
    need = kda.kda_chunk_fwd_segmented_workspace_bytes(1, T, H, 128, 128, 64, torch.bfloat16, 3)
    assert need > kda.kda_chunk_fwd_segmented_workspace_bytes(1, T, H, 128, 128, 64,
                                                              torch.bfloat16, 0)
    q, k, v = _vp(0x100000), _vp(0x200000), _vp(0x300000)
    g, beta, o = _vp(0x400000), _vp(0x800000), _vp(0x900000)
    ws = _vp(0x1000000)
    args = (q, k, v, g, beta, 1.0, None, None, 1, T, H, 128, 128, 64, 1, o, None)
    st = L.kda_chunk_fwd_segmented_ws(*args, -1, ws, need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"negative" in L.kda_last_error()
    st = L.kda_chunk_fwd_segmented_ws(*args, 3, None, need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace is NULL" in L.kda_last_error()
    st = L.kda_chunk_fwd_segmented_ws(*args, 3, ws, need - 16, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace holds" in L.kda_last_error()
    f32 = (q, k, v, g, beta, 1.0, None, None, 1, T, H, 128, 128, 64, 0, o, None)
    st = L.kda_chunk_fwd_segmented_ws(*f32, 3, ws, need, None)
    assert st == kda.KDA_ERR_UNSUPPORTED


def test_chunk_fwd_windowed_workspace_and_bad_arguments(kda):
    """The windowed workspace is one window of records plus two carry states per
    head, whatever T is; argument checks run before any device call."""
    import torch
    L = kda.lib
    T, H, W = 640, 2, 3
    need = kda.kda_chunk_fwd_windowed_workspace_bytes(1, T, H, 128, 128, 64, torch.bfloat16, W)
    assert need == 1024 + W * H * 90880 + 2 * H * 128 * 128 * 4
    assert need == kda.kda_chunk_fwd_windowed_workspace_bytes(1, 100 * T, H, 128, 128, 64,
                                                              torch.bfloat16, W)
    assert kda.kda_chunk_fwd_windowed_workspace_bytes(1, T, H, 128, 128, 64, torch.bfloat16,
                                                      0) == 0
    assert kda.kda_chunk_fwd_windowed_workspace_bytes(1, T, H, 128, 128, 64, torch.float32,
                                                      W) == 0
    q, k, v = _vp(0x100000), _vp(0x200000), _vp(0x300000)
    g, beta, o = _vp(0x400000), _vp(0x800000), _vp(0x900000)
    ws = _vp(0x1000000)
    args = (q, k, v, g, beta, 1.0, None, None, 1, T, H, 128, 128, 64, 1, o, None)
    st = L.kda_chunk_fwd_windowed_ws(*args, 0, ws, need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"window_chunks" in L.kda_last_error()
    st = L.kda_chunk_fwd_windowed_ws(*args, W, None, need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace is NULL" in L.kda_last_error()
    st = L.kda_chunk_fwd_windowed_ws(*args, W, ws, need - 16, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace holds" in L.kda_last_error()
    st = L.kda_chunk_fwd_windowed_ws(*args, W, _vp(0x900000 + 4096), need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"overlaps" in L.kda_last_error()
    f32 = (q, k, v, g, beta, 1.0, None, None, 1, T, H, 128, 128, 64, 0, o, None)
    st = L.kda_chunk_fwd_windowed_ws(*f32, W, ws, need, None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    # the fused form: x [T, 3*H*128] bf16, conv weights, g, beta, o
    x, cw = _vp(0x2000000), _vp(0x3000000)
    fargs = (x, cw, None, None, g, beta, 1.0, None, None, 1, T, H, 128, 1, o, None)
    st = L.kda_prologue_chunk_fwd_windowed_ws(*fargs, 0, ws, need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"window_chunks" in L.kda_last_error()
    st = L.kda_prologue_chunk_fwd_windowed_ws(*fargs, W, None, need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace is NULL" in L.kda_last_error()
    st = L.kda_prologue_chunk_fwd_windowed_ws(*fargs, W, ws, need - 16, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace holds" in L.kda_last_error()


def test_chunk_fwd_ws_rejects_bad_workspace(kda):
    import torch
    L = kda.lib
    T, H = 128, 2
    need = kda.kda_chunk_fwd_workspace_bytes(1, T, H, 128, 128, 64, torch.bfloat16)
    q, k, v = _vp(0x10000), _vp(0x20000), _vp(0x30000)   # 64 KiB each
    g, beta, o = _vp(0x40000), _vp(0x60000), _vp(0x70000)  # 128 KiB, 1 KiB, 128 KiB
    ws = _vp(0x100000)
    st = L.kda_chunk_fwd_ws(q, k, v, g, beta, 1.0, None, None, 1, T, H, 128, 128, 64, 1, o,
                            None, ws, need - 16, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace holds" in L.kda_last_error()
    st = L.kda_chunk_fwd_ws(q, k, v, g, beta, 1.0, None, None, 1, T, H, 128, 128, 64, 1, o,
                            None, _vp(0x100008), need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"aligned" in L.kda_last_error()
    st = L.kda_chunk_fwd_ws(q, k, v, g, beta, 1.0, None, None, 1, T, H, 128, 128, 64, 1, o,
                            None, _vp(0x78000), need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace overlaps" in L.kda_last_error()


def test_chunk_fwd_static_rejects_sizes_beyond_its_buffer(kda):
    """Checked on the host before anything is launched (fake pointers are never
    touched): T=32768, H=8 needs more than the fixed 64 MiB scratch."""
    import torch
    L = kda.lib
    T, H = 32768, 8
    assert kda.kda_chunk_fwd_workspace_bytes(1, T, H, 128, 128, 64, torch.bfloat16) > \
        kda.KDA_CHUNK_STATIC_SCRATCH_BYTES
    step = 0x10000000  # 256 MiB apart: no two fake arrays overlap
    q, k, v, g, beta, o = (_vp(step * i) for i in range(1, 7))
    st = L.kda_chunk_fwd_static(q, k, v, g, beta, 1.0, None, None, 1, T, H, 128, 128, 64, 1, o,
                                None, None)
    assert st == kda.KDA_ERR_UNSUPPORTED and b"static buffer holds" in L.kda_last_error()


def test_static_scratch_constant_matches_header(kda):
    text = open(HEADER).read()
    m = re.search(r"#define KDA_CHUNK_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == kda.KDA_CHUNK_STATIC_SCRATCH_BYTES


def test_library_sources_never_allocate_device_memory():
    """The status word and the static scratch are file-scope __device__
    variables; no source of the library calls an allocator."""
    csrc = os.path.join(ROOT, "gated_delta_rule_prologue_b200", "csrc")
    banned = re.compile(r"\b(cudaMalloc\w*|cudaFree\w*|cuMemAlloc\w*|cuMemCreate|"
                        r"cudaHostAlloc|cudaMallocHost)\b")
    for f in sorted(os.listdir(csrc)):
        src = open(os.path.join(csrc, f), encoding="utf-8").read()
        src = re.sub(r"//[^\n]*|/\*.*?\*/", "", src, flags=re.S)  # code only
        assert not banned.search(src), (f, banned.search(src).group(0))
    for f, sym in (("kda_status.cu", "g_status_word"), ("kda_static.cu", "g_static_scratch")):
        src = open(os.path.join(csrc, f), encoding="utf-8").read()
        assert re.search(r"__device__[^;]*\b%s\b" % sym, src), f
        assert "cudaGetSymbolAddress" in src, f


def test_gated_entry_points_reject_bad_gate_arguments(kda):
    L = kda.lib
    T, H = 128, 2
    need = kda.kda_chunk_fwd_workspace_bytes(1, T, H, 128, 128, 64, __import__("torch").bfloat16)
    q, k, v = _vp(0x10000), _vp(0x20000), _vp(0x30000)   # 64 KiB each
    g_raw, beta, o = _vp(0x40000), _vp(0x60000), _vp(0x70000)
    ws = _vp(0x100000)
    # lower bound below the chunk kernels' decay range
    st = L.kda_chunk_fwd_gated_ws(q, k, v, g_raw, None, None, -6.0, beta, 1.0, None, None, 1, T, H,
                                  128, 128, 64, 1, o, None, ws, need, None)
    assert st == kda.KDA_ERR_UNSUPPORTED and b"lower_bound" in L.kda_last_error()
    # non-negative lower bound
    st = L.kda_chunk_fwd_gated_ws(q, k, v, g_raw, None, None, 0.0, beta, 1.0, None, None, 1, T, H,
                                  128, 128, 64, 1, o, None, ws, need, None)
    assert st == kda.KDA_ERR_INVALID_ARG
    # one-pass shapes are not supported by the gated path
    st = L.kda_chunk_fwd_gated_ws(q, k, v, g_raw, None, None, -5.0, beta, 1.0, None, None, 1, T, H,
                                  128, 128, 32, 1, o, None, ws, need, None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    # a workspace is required
    st = L.kda_chunk_fwd_gated_ws(q, k, v, g_raw, None, None, -5.0, beta, 1.0, None, None, 1, T, H,
                                  128, 128, 64, 1, o, None, None, 0, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace" in L.kda_last_error()
    # misaligned dt_bias
    st = L.kda_decode_step_gated(q, _vp(0x200000), _vp(0x300000), g_raw, None, _vp(0x400008), -5.0,
                                 beta, 1.0, _vp(0x500000), 1, H, 128, 1, o, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"dt_bias" in L.kda_last_error()


def test_output_epilogue_rejects_bad_arguments(kda):
    L = kda.lib
    o, g, w, out = _vp(0x100000), _vp(0x200000), _vp(0x300000), _vp(0x400000)
    st = L.kda_output_epilogue(o, g, w, 1e-5, 10, 2, 48, 1, out, None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    st = L.kda_output_epilogue(o, g, w, -1.0, 10, 2, 128, 1, out, None)
    assert st == kda.KDA_ERR_INVALID_ARG
    st = L.kda_output_epilogue(o, g, None, 1e-5, 10, 2, 128, 1, out, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"weight" in L.kda_last_error()
    st = L.kda_output_epilogue(o, g, w, 1e-5, 10, 2, 128, 1, _vp(0x100010), None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"overlaps" in L.kda_last_error()


def test_chunk_map_and_compose_reject_bad_arguments(kda):
    import torch
    L = kda.lib
    T, H = 200, 2
    need = L.kda_chunk_map_workspace_bytes(1, T, H, 128, 128, 64, 1)
    assert need == kda.kda_chunk_fwd_segmented_workspace_bytes(1, T, H, 128, 128, 64,
                                                                torch.bfloat16, 0)
    assert L.kda_chunk_map_workspace_bytes(1, T, H, 128, 128, 64, 0) == 0
    q, k, v = _vp(0x100000), _vp(0x200000), _vp(0x300000)
    g, beta = _vp(0x400000), _vp(0x800000)
    M, B, ws = _vp(0x1000000), _vp(0x1100000), _vp(0x2000000)
    args = (q, k, v, g, beta, None, 1, T, H, 128, 128, 64)
    st = L.kda_chunk_map_ws(*args, 0, M, B, ws, need, None)           # f32: no tensor cores
    assert st == kda.KDA_ERR_UNSUPPORTED
    st = L.kda_chunk_map_ws(*args, 1, None, B, ws, need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"M is NULL" in L.kda_last_error()
    st = L.kda_chunk_map_ws(*args, 1, M, M, ws, need, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"overlaps" in L.kda_last_error()
    st = L.kda_chunk_map_ws(*args, 1, M, B, ws, need - 16, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"workspace holds" in L.kda_last_error()
    E = _vp(0x1200000)
    assert L.kda_state_compose(M, B, E, _vp(0x1300000), 1, 2, 64, None) == kda.KDA_ERR_UNSUPPORTED
    st = L.kda_state_compose(M, B, E, E, 1, 2, 128, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"E_out overlaps" in L.kda_last_error()
    st = L.kda_state_compose(M, None, E, _vp(0x1300000), 1, 2, 128, None)
    assert st == kda.KDA_ERR_INVALID_ARG and b"B is NULL" in L.kda_last_error()
