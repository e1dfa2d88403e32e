"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function the header declares, sizes things as documented, and rejects
bad arguments before touching CUDA."""
import ctypes

import pytest

from trellis_coded_weight_tcq_b200 import tcq


@pytest.fixture(scope="module")
def lib():
    from trellis_coded_weight_tcq_b200 import build

    build.build()
    return tcq.load_library()


def test_every_declared_function_is_exported(lib):
    names = tcq.header_functions()
    assert set(names) >= {"tcq_encode", "tcq_decode", "tcq_encode_workspace_bytes",
                          "tcq_words_per_block", "tcq_status_string", "tcq_encode_path"}
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/tcq.h but not exported"


def test_binding_signatures_match_header(lib):
    """Every declared function has ctypes argtypes with one entry per C parameter
    (a missing declaration would pass 64-bit arguments as 32-bit ints)."""
    import re

    with open(tcq.HEADER_PATH) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    tcq._static_scratch_fn()
    for name in tcq.header_functions():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)", text)
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        fn = getattr(lib, name)
        assert fn.argtypes is not None, f"{name}: binding sets no argtypes"
        assert len(fn.argtypes) == len(params), f"{name}: {len(fn.argtypes)} != {len(params)}"
        for c_param, py_type in zip(params, fn.argtypes):
            if "int64_t" in c_param or "size_t" in c_param:
                assert ctypes.sizeof(py_type) == 8, f"{name}: {c_param.strip()} must be 64-bit"


def test_words_per_block(lib):
    assert tcq.tcq_words_per_block(2, 256) == 16
    assert tcq.tcq_words_per_block(3, 256) == 24
    assert tcq.tcq_words_per_block(2, 64) == 4
    assert tcq.tcq_words_per_block(3, 11) == 2
    assert tcq.tcq_words_per_block(1, 1) == 1
    assert tcq.tcq_words_per_block(0, 5) == -1
    assert tcq.tcq_words_per_block(5, 5) == -1
    assert tcq.tcq_words_per_block(2, 0) == -1


def test_status_strings(lib):
    for s in range(6):
        assert tcq.tcq_status_string(s).startswith("TCQ_")
    assert "unknown" in tcq.tcq_status_string(99)


def test_encode_path_names(lib):
    assert tcq.tcq_encode_path(16, 2, tcq.TCQ_F16).startswith("grouped<16,2")
    assert tcq.tcq_encode_path(16, 3, tcq.TCQ_F16).startswith("grouped<16,3")
    assert tcq.tcq_encode_path(12, 2, tcq.TCQ_F32).startswith("grouped<12,2")
    assert tcq.tcq_encode_path(8, 2, tcq.TCQ_F32) == "warp<8,2>"  # blocks of up to 1024 steps
    assert tcq.tcq_encode_path(8, 2, tcq.TCQ_F16) == "warp<8,2>"
    assert tcq.tcq_encode_path(16, 2, tcq.TCQ_F32) == "generic"
    assert tcq.tcq_encode_path(3, 2, tcq.TCQ_F16) == "generic"
    assert tcq.tcq_encode_path(17, 2, tcq.TCQ_F32) == "unsupported"
    assert tcq.tcq_encode_path(8, 0, tcq.TCQ_F32) == "unsupported"
    assert tcq.tcq_encode_path(8, 2, 7) == "unsupported"


def test_workspace_query(lib):
    F16, F32 = tcq.TCQ_F16, tcq.TCQ_F32
    assert tcq.tcq_encode_workspace_bytes(16, 2, 256, 0, F16) == 0
    assert tcq.tcq_encode_workspace_bytes(17, 2, 256, 10, F16) == 0
    assert tcq.tcq_encode_workspace_bytes(8, 9, 256, 10, F32) == 0
    assert tcq.tcq_encode_workspace_bytes(8, 2, 256, 10, 5) == 0
    one = tcq.tcq_encode_workspace_bytes(16, 2, 256, 1, F16)
    # one CTA: two round buffers of (T-1) steps x 512 threads x 8 bytes of
    # backpointers, plus the traced path (T states of 2 bytes)
    assert one == 2 * ((255 * 512 * 8 + 255) // 256 * 256) + 512
    many = tcq.tcq_encode_workspace_bytes(16, 2, 256, 10**6, F16)
    assert many >= one and many % one == 0
    # the generic kernel (fp32 codebook at L=16): one byte per (step, u) plus
    # path metrics in global memory
    assert tcq.tcq_encode_workspace_bytes(16, 2, 256, 1, F32) == 255 * 16384 + 2 * 4 * 16384
    assert tcq.tcq_encode_workspace_bytes(4, 4, 1, 3, F32) == 0  # T = 1 needs no backpointers


def test_rejections_happen_before_cuda(lib):
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: every call below is rejected on the host
    vals = dict(x=fake, d=None, cb=fake, dt=tcq.TCQ_F32, L=8, k=2, T=16, n=4, st=fake, bits=fake,
                cost=fake, ws=fake, wsb=1 << 20, stream=None)

    def call(**over):
        v = dict(vals, **over)
        return tcq.tcq_encode(v["x"], v["d"], v["cb"], v["dt"], v["L"], v["k"], v["T"], v["n"],
                              v["st"], v["bits"], v["cost"], v["ws"], v["wsb"], v["stream"])

    assert call(n=0, x=None, cb=None, st=None, bits=None, cost=None, ws=None) == tcq.TCQ_OK
    assert call(n=-1) == tcq.TCQ_ERR_INVALID_ARG
    assert call(x=None) == tcq.TCQ_ERR_INVALID_ARG
    assert call(ws=None) == tcq.TCQ_ERR_INVALID_ARG
    assert call(x=ctypes.c_void_p(0x10002)) == tcq.TCQ_ERR_INVALID_ARG
    assert call(ws=ctypes.c_void_p(0x10010)) == tcq.TCQ_ERR_INVALID_ARG
    assert call(dt=3) == tcq.TCQ_ERR_INVALID_ARG
    assert call(L=17) == tcq.TCQ_ERR_UNSUPPORTED
    assert call(L=1, k=2) == tcq.TCQ_ERR_UNSUPPORTED
    assert call(k=5, L=8) == tcq.TCQ_ERR_UNSUPPORTED
    assert call(T=0) == tcq.TCQ_ERR_UNSUPPORTED
    assert call(T=(1 << 20) + 1) == tcq.TCQ_ERR_UNSUPPORTED
    dec = lambda **o: tcq.tcq_decode(o.get("bits", fake), o.get("st", fake), o.get("cb", fake),  # noqa: E731
                                     o.get("dt", 0), o.get("L", 8), o.get("k", 2), o.get("T", 16),
                                     o.get("n", 4), o.get("y", fake), None)
    assert dec(n=0, bits=None, st=None, cb=None, y=None) == tcq.TCQ_OK
    assert dec(y=None) == tcq.TCQ_ERR_INVALID_ARG
    assert dec(bits=ctypes.c_void_p(0x10001)) == tcq.TCQ_ERR_INVALID_ARG
    assert dec(dt=1, cb=ctypes.c_void_p(0x10001)) == tcq.TCQ_ERR_INVALID_ARG
    assert dec(L=0) == tcq.TCQ_ERR_UNSUPPORTED
    assert dec(n=-5) == tcq.TCQ_ERR_INVALID_ARG


def test_binding_rejects_undersized_tensors_before_any_launch():
    """The Python wrappers check tensor sizes against the shape they are given,
    so a call can never hand the library a buffer smaller than the matrix."""
    import torch
    from trellis_coded_weight_tcq_b200 import tcq

    W = tcq.tcq_words_per_block(2, 256)
    bits = torch.zeros((10, W), dtype=torch.int32)
    start = torch.zeros(10, dtype=torch.int32)
    cb = torch.zeros(1 << 16, dtype=torch.float16)
    x = torch.zeros(4096)
    with pytest.raises(ValueError):  # 74 x 4096 needs 1184 blocks
        tcq.gemv(bits, start, None, cb, 16, 2, 256, 74, 4096, x)
    with pytest.raises(ValueError):
        tcq.decode(bits[:5], start, cb, 16, 2, 256)
    with pytest.raises(ValueError):
        tcq.decode(bits, start, cb, 16, 2, 256, out=torch.empty((9, 256)))


def test_vector_and_feedback_entry_points_reject_on_the_host(lib):
    """The vector-trellis calls validate shapes, dtypes and pointers before any
    CUDA call; their workspace query covers the compile-time kernel."""
    fake = ctypes.c_void_p(0x10000)
    F16, F32 = tcq.TCQ_F16, tcq.TCQ_F32
    # the L=16, k=2, V=2 compile-time encoder: two round buffers of (T/2 - 1)
    # steps x 512 words, plus the traced path; never less than the runtime kernel needs
    one = tcq.tcq_encode_vec_workspace_bytes(16, 2, 2, 256, 1, F16)
    vec2 = 2 * ((127 * 512 * 4 + 255) // 256 * 256) + 256
    generic = tcq.tcq_encode_vec_workspace_bytes(16, 2, 2, 256, 1, F32)
    assert one >= vec2 and one >= generic
    assert tcq.tcq_encode_vec_workspace_bytes(16, 2, 2, 255, 1, F16) == 0  # V does not divide T
    assert tcq.tcq_encode_vec_workspace_bytes(16, 2, 2, 256, 1, tcq.TCQ_MAD) == 0
    gv = lambda **o: tcq.tcq_gemv_vec(o.get("bits", fake), o.get("st", fake), None,  # noqa: E731
                                      o.get("cb", fake), o.get("dt", F16), o.get("L", 16),
                                      o.get("k", 2), o.get("V", 2), o.get("T", 256),
                                      o.get("rows", 4), o.get("cols", 1024), o.get("x", fake),
                                      o.get("y", fake), None)
    assert gv(rows=0) == tcq.TCQ_OK
    assert gv(rows=-1) == tcq.TCQ_ERR_INVALID_ARG
    assert gv(cols=1000) == tcq.TCQ_ERR_INVALID_ARG                  # cols % T
    assert gv(x=ctypes.c_void_p(0x10004)) == tcq.TCQ_ERR_INVALID_ARG  # x not 16-byte aligned
    assert gv(y=None) == tcq.TCQ_ERR_INVALID_ARG
    assert gv(dt=tcq.TCQ_MAD, cb=None) == tcq.TCQ_ERR_UNSUPPORTED
    assert gv(k=3, V=3) == tcq.TCQ_ERR_UNSUPPORTED                   # kV = 9 bits per step
    dv = lambda **o: tcq.tcq_decode_vec(o.get("bits", fake), o.get("st", fake), o.get("cb", fake),  # noqa: E731
                                        o.get("dt", F16), 16, 2, o.get("V", 2), o.get("T", 256),
                                        o.get("n", 4), o.get("y", fake), None)
    assert dv(n=0) == tcq.TCQ_OK
    assert dv(T=255) == tcq.TCQ_ERR_UNSUPPORTED
    assert dv(y=ctypes.c_void_p(0x10002)) == tcq.TCQ_ERR_INVALID_ARG


def test_set_partitioned_trellis_entry_points_reject_on_the_host(lib):
    """tcq_ub8_*: sizes as documented, shapes and pointers refused before any CUDA call."""
    fake = ctypes.c_void_p(0x10000)
    F16, F32 = tcq.TCQ_F16, tcq.TCQ_F32
    assert tcq.tcq_ub8_words_per_block(4, 7, 256) == 16        # 64 steps x 8 bits
    assert tcq.tcq_ub8_words_per_block(1, 1, 100) == 7         # 100 steps x 2 bits
    assert tcq.tcq_ub8_words_per_block(3, 0, 9) == 1
    assert tcq.tcq_ub8_words_per_block(8, 8, 4096) == 144      # 512 steps x 9 bits
    assert tcq.tcq_ub8_words_per_block(4, 7, 255) == -1       # V does not divide T
    assert tcq.tcq_ub8_words_per_block(9, 1, 9) == -1
    assert tcq.tcq_ub8_words_per_block(1, 9, 8) == -1
    assert tcq.tcq_ub8_words_per_block(1, 1, 513) == -1        # more than 512 steps
    assert tcq.tcq_ub8_words_per_block(0, 1, 8) == -1

    def enc(**o):
        return tcq.tcq_ub8_encode(o.get("x", fake), o.get("d", None), o.get("cb", fake),
                                  o.get("dt", F32), o.get("V", 4), o.get("m", 7), o.get("T", 256),
                                  o.get("n", 4), o.get("fs", None), o.get("st", fake),
                                  o.get("bits", fake), o.get("cost", fake), None)

    assert enc(n=0, x=None, cb=None, st=None, bits=None, cost=None) == tcq.TCQ_OK
    assert enc(n=-1) == tcq.TCQ_ERR_INVALID_ARG
    assert enc(x=None) == tcq.TCQ_ERR_INVALID_ARG
    assert enc(cost=None) == tcq.TCQ_ERR_INVALID_ARG
    assert enc(x=ctypes.c_void_p(0x10002)) == tcq.TCQ_ERR_INVALID_ARG
    assert enc(fs=ctypes.c_void_p(0x10001)) == tcq.TCQ_ERR_INVALID_ARG
    assert enc(dt=F16, cb=ctypes.c_void_p(0x10001)) == tcq.TCQ_ERR_INVALID_ARG
    assert enc(dt=tcq.TCQ_MAD, cb=None) == tcq.TCQ_ERR_UNSUPPORTED
    assert enc(dt=7) == tcq.TCQ_ERR_INVALID_ARG
    assert enc(T=254) == tcq.TCQ_ERR_UNSUPPORTED
    assert enc(V=9, T=261) == tcq.TCQ_ERR_UNSUPPORTED
    assert enc(m=9) == tcq.TCQ_ERR_UNSUPPORTED
    assert enc(V=1, T=600) == tcq.TCQ_ERR_UNSUPPORTED

    def dec(**o):
        return tcq.tcq_ub8_decode(o.get("bits", fake), o.get("st", fake), o.get("cb", fake),
                                  o.get("dt", F32), o.get("V", 4), o.get("m", 7), o.get("T", 256),
                                  o.get("n", 4), o.get("y", fake), None)

    assert dec(n=0, bits=None, st=None, cb=None, y=None) == tcq.TCQ_OK
    assert dec(y=None) == tcq.TCQ_ERR_INVALID_ARG
    assert dec(st=ctypes.c_void_p(0x10002)) == tcq.TCQ_ERR_INVALID_ARG
    assert dec(m=-1) == tcq.TCQ_ERR_UNSUPPORTED
    assert dec(dt=tcq.TCQ_MAD, cb=None) == tcq.TCQ_ERR_UNSUPPORTED
    assert dec(n=-3) == tcq.TCQ_ERR_INVALID_ARG


def test_debug_build_exports_every_declared_function(lib):
    """The bounds-checked build compiles (sm_100a, relocatable device code) and
    exports the same C ABI; checked in a process of its own, since one process
    loads only one build of the library."""
    import os
    import subprocess
    import sys

    from trellis_coded_weight_tcq_b200 import build

    path = build.build(debug=True)
    code = ("import ctypes, sys; sys.path.insert(0, %r); "
            "from trellis_coded_weight_tcq_b200 import tcq; "
            "assert tcq.LIB_PATH.endswith('libtcq_debug.so'); lib = tcq.load_library(); "
            "missing = [n for n in tcq.header_functions() if not hasattr(lib, n)]; "
            "assert not missing, missing; print('exports ok')" % build.ROOT)
    r = subprocess.run([sys.executable, "-c", code], env=dict(os.environ, TCQ_LIBRARY="debug"),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "exports ok" in r.stdout, r.stderr[-2000:]
    assert os.path.exists(path)


@pytest.mark.parametrize("n,chunks", [(1, 8), (7, 8), (301, 1), (301, 3), (301, 8), (75775, 8),
                                      (75776, 8), (229376, 8), (1000003, 8), (5000, 16)])
def test_host_pipeline_parts(n, chunks):
    """The end-to-end pipeline's parts cover the blocks once, in order; a lead
    part then `chunks` parts (one part for chunks = 1); for large inputs every
    part but the last is a whole number of waves (8 x 148 blocks)."""
    parts = tcq.host_pipeline_parts(n, chunks, 148)
    assert parts[0][0] == 0 and parts[-1][1] == n
    assert all(hi > lo for lo, hi in parts)
    assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
    assert len(parts) == (1 if chunks == 1 else min(chunks + 1, n))
    wave = 8 * 148
    if n >= 8 * chunks * wave:
        assert all((hi - lo) % wave == 0 for lo, hi in parts[:-1])
    if chunks > 1 and len(parts) > 2:  # the lead part is the short one
        assert parts[0][1] - parts[0][0] <= min(hi - lo for lo, hi in parts[1:-1])
