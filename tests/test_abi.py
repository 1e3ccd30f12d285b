"""C ABI: the library loads, exports what include/fmoe.h declares, packs and
unpacks bit-exactly, and rejects bad arguments on the host before launching
anything (none of these tests needs a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fm():
    # the builder by its path: importing the package needs the library it builds
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fmoe_library_build", os.path.join(ROOT, "quantized_expert_gemv_b200", "build.py"))
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build()
    import quantized_expert_gemv_b200 as m
    return m


def declared_symbols():
    out = set()
    for name in os.listdir(os.path.join(ROOT, "include")):
        if name.endswith(".h"):
            src = open(os.path.join(ROOT, "include", name)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            out |= set(re.findall(r"\b(fmoe_\w+)\s*\(", src))
    return out


def test_every_declared_symbol_is_exported(fm):
    lib = ctypes.CDLL(fm.LIBRARY_PATH)
    syms = declared_symbols()
    assert len(syms) >= 15
    for s in syms:
        assert hasattr(lib, s), s
    assert syms <= set(fm.EXPORTED) | {"fmoe_error_string"}


def test_packed_bytes_closed_form(fm):
    assert fm.fmoe_packed_bytes(4, 1, 4096, 1024) == 7_077_888  # 6.75 MiB
    assert fm.fmoe_packed_bytes(2, 1, 4096, 1024) == 3_932_160  # 3.75 MiB
    assert fm.fmoe_packed_bytes(4, 512, 4096, 1024) == 512 * 7_077_888
    assert fm.fmoe_packed_bytes(4, 1, 256, 128) == 3 * 256 * 128 // 2 + 3 * 256 * 128 // 64 * 4
    # unsupported: group != 64, width not a multiple of 64, 48 groups, bits 3
    assert fm.fmoe_packed_bytes(4, 1, 4096, 1024, group=128) == 0
    assert fm.fmoe_packed_bytes(4, 1, 4000, 1024) == 0
    assert fm.fmoe_packed_bytes(4, 1, 3072, 1024) == 0
    assert fm.fmoe_packed_bytes(3, 1, 4096, 1024) == 0


@pytest.mark.parametrize("bits,H,I", [(4, 256, 128), (2, 256, 128), (4, 4096, 1024), (2, 4096, 1024),
                                      (4, 64, 2048), (2, 128, 64)])
def test_pack_unpack_round_trip(fm, bits, H, I):
    wl = synth.Workload(hidden=H, inter=I, n_experts=3, bits=bits, seed=7 + bits)
    exs = [synth.expert(wl, 1, e) for e in range(2)]
    q = np.concatenate([e.q for e in exs])
    s = np.concatenate([e.scale for e in exs])
    b = np.concatenate([e.bias for e in exs])
    packed = fm.fmoe_pack_experts_host(q, s, b, bits, 2, H, I)
    assert packed.nbytes == fm.fmoe_packed_bytes(bits, 2, H, I)
    q2, s2, b2 = fm.fmoe_unpack_experts_host(packed, bits, 2, H, I)
    assert np.array_equal(q2, q) and np.array_equal(s2, s) and np.array_equal(b2, b)
    # a host buffer at an odd address gives the same bytes and unpacks the same
    raw = np.zeros(packed.nbytes + 3, np.uint8)
    odd = raw[3:]
    assert odd.ctypes.data % 4 != 0
    fm.fmoe_pack_experts_host(q, s, b, bits, 2, H, I, out=odd)
    assert np.array_equal(odd, packed)
    q3, s3, b3 = fm.fmoe_unpack_experts_host(odd, bits, 2, H, I)
    assert np.array_equal(q3, q) and np.array_equal(s3, s) and np.array_equal(b3, b)


@pytest.mark.parametrize("bits", [4, 2])
def test_pack_extreme_codes(fm, bits):
    H, I = 128, 64
    n, ng = 3 * H * I, 3 * H * I // 64
    for fill in (0, (1 << bits) - 1):
        q = np.full(n, fill, np.uint8)
        s = np.full(ng, 0x3C00, np.uint16)  # 2^-7
        b = np.full(ng, 0xBF80, np.uint16)  # -1
        packed = fm.fmoe_pack_experts_host(q, s, b, bits, 1, H, I)
        q2, s2, b2 = fm.fmoe_unpack_experts_host(packed, bits, 1, H, I)
        assert np.array_equal(q2, q) and np.array_equal(s2, s) and np.array_equal(b2, b)


def test_packed_word_permutation(fm):
    """Inputs 0..7 of a 4-bit row land in the documented fields: field 2a+b
    of the first word holds input 4b+a."""
    H, I = 64, 64
    n, ng = 3 * H * I, 3 * H * I // 64
    q = np.zeros(n, np.uint8)
    q[:8] = [1, 2, 3, 4, 5, 6, 7, 8]  # gate row 0, inputs 0..7
    s = np.full(ng, 0x3F80, np.uint16)
    b = np.zeros(ng, np.uint16)
    packed = fm.fmoe_pack_experts_host(q, s, b, 4, 1, H, I)
    word = int(packed[:4].view(np.uint32)[0])
    fields = [(word >> (4 * p)) & 0xF for p in range(8)]
    for a in range(4):
        for bb in range(2):
            assert fields[2 * a + bb] == q[4 * bb + a]
    # scale is stored pre-multiplied by 2^-4: 1.0 -> 0x3D80
    sb_off = 2 * 64 * H * 4 // 8 + H * I * 4 // 8
    assert int(packed[sb_off:sb_off + 4].view(np.uint32)[0]) & 0xFFFF == 0x3D80


@pytest.mark.parametrize("bits", [4, 2])
def test_packed_down_column_blocks(fm, bits):
    """Down codes are stored column block by column block: the word at
    (block nb, row r) holds inputs nb*w .. nb*w + w - 1 of down row r (w = 32 /
    bits) in the documented field order; down scale-bias words are group-major."""
    H, I = 128, 128
    n, ng = H * I, H * I // 64
    rng = np.random.default_rng(bits)
    q = rng.integers(0, 1 << bits, size=3 * n, dtype=np.uint8)
    s = np.full(3 * ng, 0x3F80, np.uint16)
    b = rng.integers(0, 1 << 15, size=3 * ng).astype(np.uint16)
    packed = fm.fmoe_pack_experts_host(q, s, b, bits, 1, H, I)
    w, per_byte = 32 // bits, 8 // bits
    down_codes = 2 * I * H * bits // 8
    words = packed[down_codes:down_codes + H * I * bits // 8].view(np.uint32)
    qd = q[2 * n:].reshape(H, I)
    for nb, r in [(0, 0), (1, 5), (I // w - 1, H - 1), (3, 77)]:
        word = int(words[nb * H + r])
        for a in range(4):
            for bb in range(per_byte):
                field = (word >> (bits * (per_byte * a + bb))) & ((1 << bits) - 1)
                assert field == qd[r, nb * w + 4 * bb + a]
    sb_off = down_codes + H * I * bits // 8 + 2 * I * (H // 64) * 4
    sbw = packed[sb_off:sb_off + H * (I // 64) * 4].view(np.uint32)
    bd = b[2 * ng:].reshape(H, I // 64)
    for g, r in [(0, 0), (1, 3), (I // 64 - 1, H - 1)]:
        assert int(sbw[g * H + r]) >> 16 == bd[r, g]


def test_packer_rejects_bad_input(fm):
    H, I = 64, 64
    n, ng = 3 * H * I, 3 * H * I // 64
    q = np.zeros(n, np.uint8)
    s = np.full(ng, 0x3F80, np.uint16)
    b = np.zeros(ng, np.uint16)
    q[5] = 16  # out of range for 4-bit
    with pytest.raises(fm.FmoeError) as e:
        fm.fmoe_pack_experts_host(q, s, b, 4, 1, H, I)
    assert e.value.status == fm.FMOE_ERR_INVALID_ARG
    q[5] = 4
    with pytest.raises(fm.FmoeError):
        fm.fmoe_pack_experts_host(q, s, b, 2, 1, H, I)  # 4 > 3 for 2-bit
    s[3] = 0x0001  # subnormal scale cannot be pre-scaled exactly
    q[5] = 0
    with pytest.raises(fm.FmoeError):
        fm.fmoe_pack_experts_host(q, s, b, 4, 1, H, I)
    with pytest.raises(fm.FmoeError) as e:
        fm.fmoe_pack_experts_host(q, s, b, 4, 1, 96, 64)
    assert e.value.status == fm.FMOE_ERR_UNSUPPORTED


H_, XN_ = 1 << 20, (1 << 20) + 1024  # distinct device addresses of one 256-float token row each


def test_host_validation_before_launch(fm):
    """Bad arguments are refused on the host (no CUDA call is made, so this
    runs without a GPU)."""
    L = fm._lib
    assert L.fmoe_layer_forward(None, None, None, 1, None, 0, None) == fm.FMOE_ERR_INVALID_ARG
    d = fm.LayerDesc(hidden=256, inter=128, n_experts=16, top_k=4)
    w = fm.fmoe_layer_weights(d.c(), 16, 16, 16, 16, 16)
    # null activation pointers
    assert L.fmoe_layer_forward(ctypes.byref(w), None, None, 1, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    # misaligned workspace
    assert L.fmoe_layer_forward(ctypes.byref(w), H_, XN_, 1, 17, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    # workspace too small
    assert L.fmoe_layer_forward(ctypes.byref(w), H_, XN_, 1, 16, 64, None) == fm.FMOE_ERR_BUFFER_TOO_SMALL
    # h and xn overlapping (one token of H = 256 floats is 1 KiB): refused,
    # rows that only touch are not
    for xn in (H_, H_ + 1008, H_ - 1008):
        assert L.fmoe_layer_forward(ctypes.byref(w), H_, xn, 1, 16, 64, None) == fm.FMOE_ERR_INVALID_ARG
        assert L.fmoe_layer_forward_logits(ctypes.byref(w), 16, H_, xn, 1, 16, 64, None) == fm.FMOE_ERR_INVALID_ARG
        assert L.fmoe_stack_forward(ctypes.byref(w), 1, H_, xn, 1, 16, 64, None) == fm.FMOE_ERR_INVALID_ARG
        assert L.fmoe_layer_forward_noalloc(ctypes.byref(w), H_, xn, 1, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_layer_forward(ctypes.byref(w), H_, XN_, 2, 16, 64, None) == fm.FMOE_ERR_INVALID_ARG  # 2 tokens
    for xn in (H_ + 1024, H_ - 1024):
        assert L.fmoe_layer_forward(ctypes.byref(w), H_, xn, 1, 16, 64, None) == fm.FMOE_ERR_BUFFER_TOO_SMALL
    # k > 8, k > E, E > 1024, T < 1
    for bad in (dict(top_k=9, n_experts=16), dict(top_k=5, n_experts=4), dict(n_experts=2048)):
        dd = fm.LayerDesc(hidden=256, inter=128, **{**dict(n_experts=16, top_k=4), **bad})
        ww = fm.fmoe_layer_weights(dd.c(), 16, 16, 16, 16, 16)
        assert L.fmoe_layer_forward(ctypes.byref(ww), 16, 16, 1, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_layer_forward(ctypes.byref(w), 16, 16, 0, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    # unsupported shapes / bits
    for bad in (dict(hidden=96), dict(inter=3072), dict(bits=3), dict(shared_bits=8), dict(group=32)):
        dd = fm.LayerDesc(**{**dict(hidden=256, inter=128, n_experts=16, top_k=4), **bad})
        ww = fm.fmoe_layer_weights(dd.c(), 16, 16, 16, 16, 16)
        assert L.fmoe_layer_forward(ctypes.byref(ww), 16, 16, 1, 16, 1 << 30, None) == fm.FMOE_ERR_UNSUPPORTED
    # expert forward: k mismatch
    assert L.fmoe_expert_forward(ctypes.byref(w), 16, 1, 16, 3, 16, 16, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    # route: k > 8 unsupported, null outputs invalid
    assert L.fmoe_route_topk(16, 16, 1, 256, 16, 9, 0, 16, 16, 16, 16, 1 << 20, None) == fm.FMOE_ERR_UNSUPPORTED
    assert L.fmoe_route_topk(16, 16, 1, 256, 16, 4, 0, None, 16, 16, 16, 1 << 20, None) == fm.FMOE_ERR_INVALID_ARG
    # combine: an output overlapping an input or the other output (one
    # token of H = 256: rows of 1 KiB, y of 5 KiB); h_out = h is in place
    Y = 1 << 24
    comb = lambda y, h, ho, xo: L.fmoe_combine_residual_rmsnorm(y, 16, 16, h, 16, ctypes.c_float(1e-6), 1, 4, 256,
                                                                ho, xo, None)
    assert comb(Y, 32, 32, 32) == fm.FMOE_ERR_INVALID_ARG            # xn_out = h
    assert comb(Y, H_, XN_, XN_) == fm.FMOE_ERR_INVALID_ARG          # xn_out = h_out
    assert comb(Y, H_, H_, Y + 4096) == fm.FMOE_ERR_INVALID_ARG      # xn_out inside y
    assert comb(Y, H_, Y - 512, XN_) == fm.FMOE_ERR_INVALID_ARG      # h_out runs into y
    assert comb(Y, H_, H_ + 512, XN_ + 1024) == fm.FMOE_ERR_INVALID_ARG  # h_out half over h
    assert L.fmoe_stack_forward(None, 1, 16, 16, 1, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_error_string(fm.FMOE_ERR_UNSUPPORTED) == "unsupported shape or bit width"


def test_host_validation_of_the_later_entry_points(fm):
    """Quantiser, host-state layer forward and expert cache refuse bad
    arguments on the host, before any CUDA call (runs without a GPU)."""
    L = fm._lib
    # quantiser: null / misaligned pointers, group and bit width, empty input
    assert L.fmoe_quantize_groups(None, 4, 64, 4, 16, 16, 16, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_quantize_groups(16, 4, 64, 4, 24, 16, 16, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_quantize_groups(16, 4, 32, 4, 16, 16, 16, None) == fm.FMOE_ERR_UNSUPPORTED
    assert L.fmoe_quantize_groups(16, 4, 64, 3, 16, 16, 16, None) == fm.FMOE_ERR_UNSUPPORTED
    assert L.fmoe_quantize_groups(16, 0, 64, 2, 16, 16, 16, None) == fm.FMOE_OK
    # host-state layer forward: null buffers, workspace too small
    d = fm.LayerDesc(hidden=256, inter=128, n_experts=16, top_k=4)
    w = fm.fmoe_layer_weights(d.c(), 16, 16, 16, 16, 16)
    assert L.fmoe_layer_forward_host(ctypes.byref(w), None, 16, 16, 1, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_layer_forward_host(ctypes.byref(w), 16, 16, 24, 1, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_layer_forward_host(ctypes.byref(w), 16, 16, 16, 1, 16, 64, None) == fm.FMOE_ERR_BUFFER_TOO_SMALL
    # host-state stack: no layers, null buffers, workspace too small
    ws2 = (fm.fmoe_layer_weights * 2)(w, w)
    assert L.fmoe_stack_forward_host(None, 1, 16, 16, 16, 1, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_stack_forward_host(ws2, 2, None, 16, 16, 1, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_stack_forward_host(ws2, 2, 16, 16, 24, 1, 16, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_stack_forward_host(ws2, 2, 16, 16, 16, 1, 16, 64, None) == fm.FMOE_ERR_BUFFER_TOO_SMALL
    # expert cache: missing arguments, slots too small for n_slots records
    dc = d.c()
    hp = (ctypes.c_void_p * 1)(16)
    out = ctypes.c_void_p()
    assert L.fmoe_cache_create(None, 1, hp, 4, 16, 1 << 30, 16, 1, ctypes.byref(out)) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_cache_create(ctypes.byref(dc), 1, None, 4, 16, 1 << 30, 16, 1, ctypes.byref(out)) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_cache_create(ctypes.byref(dc), 1, hp, 4, 16, 64, 16, 1, ctypes.byref(out)) == fm.FMOE_ERR_BUFFER_TOO_SMALL
    assert L.fmoe_cache_create(ctypes.byref(dc), 1, hp, 0, 16, 1 << 30, 16, 1, ctypes.byref(out)) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_cache_layer_forward(None, 0, ctypes.byref(w), None, 16, 16, 1, 16, 1 << 30, None) == \
        fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_cache_stats(None, None, None, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_cache_destroy(None) == fm.FMOE_ERR_INVALID_ARG
    # the dispatch thresholds the header states
    assert fm.fmoe_tc_min_tokens() == 3
    assert fm.fmoe_fused_max_tokens(False) == 4 and fm.fmoe_fused_max_tokens(True) == 8


def test_product_library_has_no_timeline_build(fm):
    """The timer reads of the per-phase timeline exist only in the separate
    FMOE_TIMELINE build (quantized_expert_gemv_b200/timeline.py)."""
    assert not hasattr(fm._lib, "fmoe_timeline_read")
    assert not hasattr(fm._lib, "fmoe_timeline_layer")


def test_workspace_layout(fm):
    d = fm.LayerDesc()
    n1, n64 = fm.fmoe_workspace_bytes(d, 1), fm.fmoe_workspace_bytes(d, 64)
    assert 0 < n1 < n64
    offs = [fm.fmoe_workspace_offset(d, 3, w) for w in range(6)]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert fm.fmoe_workspace_offset(d, 3, 6) == 2 ** 64 - 1


def test_trace_layout_and_validation(fm):
    """A stack trace: one record per layer, sections in the declared order,
    256-byte aligned, sized for T tokens; bad arguments refused on the host."""
    L = fm._lib
    d = fm.LayerDesc()
    T, n = 3, 5
    H, I, E, k = d.hidden, d.inter, d.n_experts, d.top_k
    rec = fm.fmoe_trace_bytes(d, T, 1)
    assert fm.fmoe_trace_bytes(d, T, n) == n * rec
    sizes = [T * H * 4, T * E * 4, T * k * 4, T * k * 4, T * 4, T * (k + 1) * I * 4, T * H * 4]
    dc = d.c()
    offs = [L.fmoe_trace_offset(ctypes.byref(dc), T, 2, w) for w in range(7)]
    assert all(o % 256 == 0 for o in offs)
    assert offs[0] == 2 * rec
    for w in range(6):
        assert offs[w + 1] >= offs[w] + sizes[w]
    assert 2 * rec + rec >= offs[6] + sizes[6]
    assert L.fmoe_trace_offset(ctypes.byref(dc), T, 0, 7) == 2 ** 64 - 1
    assert L.fmoe_trace_offset(ctypes.byref(dc), T, -1, 0) == 2 ** 64 - 1
    assert L.fmoe_trace_bytes(ctypes.byref(dc), 0, 1) == 0
    # trace entry point: null or misaligned trace, trace too small
    dd = fm.LayerDesc(hidden=256, inter=128, n_experts=16, top_k=4)
    w = fm.fmoe_layer_weights(dd.c(), 16, 16, 16, 16, 16)
    w2 = (fm.fmoe_layer_weights * 2)(w, w)
    assert L.fmoe_stack_forward_trace(w2, 2, H_, XN_, 1, 16, 1 << 30, None, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    assert L.fmoe_stack_forward_trace(w2, 2, H_, XN_, 1, 16, 1 << 30, 24, 1 << 30, None) == fm.FMOE_ERR_INVALID_ARG
    need = fm.fmoe_trace_bytes(dd, 1, 2)
    assert L.fmoe_stack_forward_trace(w2, 2, H_, XN_, 1, 16, 1 << 30, 16, need - 1, None) == \
        fm.FMOE_ERR_BUFFER_TOO_SMALL
    assert L.fmoe_stack_forward_trace(w2, 2, H_, H_, 1, 16, 1 << 30, 16, need, None) == fm.FMOE_ERR_INVALID_ARG


def test_header_and_c_example_compile_as_c():
    """include/fmoe.h is a C header: the plain-C example compiles with gcc
    -std=c11 against it (syntax and types only; no GPU needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if not gcc or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime.h")):
        pytest.skip("gcc or the CUDA headers are not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = os.path.join(root, "quantized_expert_gemv_b200", "examples", "decode_host.c")
    r = subprocess.run([gcc, "-std=c11", "-Wall", "-Werror", "-fsyntax-only", "-I", os.path.join(root, "include"),
                        "-I", cuda_inc, src], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_timeline_points_match_the_kernel():
    """Every timer point of the persistent kernel has a name in the timeline
    tool, and every named point is recorded somewhere in the kernel."""
    import re
    from pathlib import Path
    from quantized_expert_gemv_b200 import timeline
    src = (Path(__file__).resolve().parents[1] / "quantized_expert_gemv_b200" / "csrc" / "fmoe_fused.cuh").read_text()
    used = set()
    calls = re.findall(r"FMOE_TS\(([0-9][^)]*)\)", src)
    assert len(calls) == src.count("FMOE_TS(") - 2  # all but the two macro definitions
    for expr in calls:
        m = re.fullmatch(r"(\d+)(?: \+ p)?", expr.strip())
        assert m, expr
        base = int(m.group(1))
        used.update(range(base, base + 5) if "+ p" in expr else [base])
    assert used == set(timeline.POINTS), sorted(used ^ set(timeline.POINTS))
    assert max(used) < timeline.N_POINTS


def test_binding_refuses_bad_buffers_before_the_call(fm):
    """The Python binding checks each buffer a call reads or writes (memory
    kind, contiguity, element type, size) and raises ValueError before the
    library is called: a token buffer shorter than T x hidden, or a weight
    tensor shorter than the records the descriptor names, would otherwise be
    read or written past its end on the device.  Runs without a GPU."""
    import torch
    need = fm._need
    # host buffers: pass when right, refused for each kind of mismatch
    need(torch.zeros(4, 256), "h", 4 * 256, cuda=False)
    need(np.zeros((4, 256), np.float32), "h", 4 * 256, cuda=False)
    need(torch.zeros(3, dtype=torch.int32), "ids", 3, "i32", cuda=False)
    need(torch.zeros(100, dtype=torch.uint8), "ws", 64, None, cuda=False, exact=False)
    bad = [
        (torch.zeros(4, 255), "holds 1020 elements, the call needs 1024"),
        (torch.zeros(4, 257), "holds 1028 elements, the call needs 1024"),
        (torch.zeros(4, 256, dtype=torch.float64), "must hold float32"),
        (torch.zeros(4, 256, dtype=torch.bfloat16), "must hold float32"),
        (torch.zeros(256, 4).t(), "must be contiguous"),
        (np.zeros((4, 256), np.float64), "must hold float32"),
        (np.zeros((256, 4), np.float32).T, "must be contiguous"),
        (None, "missing"),
    ]
    for x, msg in bad:
        with pytest.raises(ValueError, match=msg):
            need(x, "h", 4 * 256, cuda=False)
    with pytest.raises(ValueError, match="at least 64"):
        need(torch.zeros(63, dtype=torch.uint8), "ws", 64, None, cuda=False, exact=False)
    with pytest.raises(ValueError, match="host memory"):
        need(torch.zeros(4, 256, device="meta"), "hx_in", 4 * 256, cuda=False)
    need(1 << 20, "h", 4 * 256)  # a raw address is the caller's own
    # device buffers given as host tensors: refused before the library is called
    d = fm.LayerDesc(hidden=256, inter=128, n_experts=16, top_k=4)
    H, E, k = d.hidden, d.n_experts, d.top_k
    lw = fm.LayerWeights(d, torch.zeros(E * d.record_bytes(), dtype=torch.uint8),
                         torch.zeros(d.record_bytes(shared=True), dtype=torch.uint8),
                         torch.zeros(E, H), torch.zeros(H), torch.ones(H))
    h, xn, ws = torch.zeros(2, H), torch.zeros(2, H), torch.zeros(1 << 20, dtype=torch.uint8)
    with pytest.raises(ValueError, match="h: must be in CUDA device memory"):
        fm.fmoe_layer_forward(lw, h, xn, ws)
    with pytest.raises(ValueError, match="h: must be in CUDA device memory"):
        fm.fmoe_stack_forward([lw, lw], h, xn, ws)
    with pytest.raises(ValueError, match="h: must be in CUDA device memory"):
        fm.fmoe_layer_forward_noalloc(lw, h, xn)
    with pytest.raises(ValueError, match="d_hx: must be in CUDA device memory"):
        fm.fmoe_layer_forward_host(lw, torch.zeros(2, 2, H), torch.zeros(2, 2, H), torch.zeros(2, 2, H), ws)
    with pytest.raises(ValueError, match="experts: must be in CUDA device memory"):
        lw.c()
    with pytest.raises(ValueError, match="y: must be in CUDA device memory"):
        fm.fmoe_combine_residual_rmsnorm(torch.zeros(2, k + 1, H), torch.zeros(2, k), torch.zeros(2), h,
                                         torch.ones(H), 1e-6, h, xn)
    with pytest.raises(ValueError, match="logits: must be in CUDA device memory"):
        fm.fmoe_route_topk(None, None, k, torch.zeros(2, E), torch.zeros(2, k, dtype=torch.int32), torch.zeros(2, k),
                           flags=fm.FMOE_LOGITS_GIVEN)
    with pytest.raises(ValueError, match="xn: must be in CUDA device memory"):
        fm.fmoe_expert_forward(lw, xn, torch.zeros(2, k, dtype=torch.int32), torch.zeros(2, k + 1, H),
                               torch.zeros(2), ws)
    # packers: the codes and scales of every expert must be there (shape
    # supported); an unsupported shape is still the library's to refuse
    q = np.zeros(3 * H * 128, np.uint8)
    sb = np.zeros(3 * H * 128 // 64, np.uint16)
    with pytest.raises(ValueError, match="q: holds"):
        fm.fmoe_pack_experts_host(q, sb, sb, 4, 2, H, 128)
    with pytest.raises(ValueError, match="scale: holds"):
        fm.fmoe_pack_experts_host(np.zeros(2 * 3 * H * 128, np.uint8), sb, sb, 4, 2, H, 128)
    with pytest.raises(ValueError, match="packed: holds"):
        fm.fmoe_unpack_experts_host(np.zeros(100, np.uint8), 4, 1, H, 128)
    with pytest.raises(ValueError, match="q: must be in CUDA device memory"):
        fm.fmoe_pack_experts_device(q, sb, sb, 4, 1, H, 128, torch.zeros(10, dtype=torch.uint8))
    with pytest.raises(ValueError, match="w: must be in CUDA device memory"):
        fm.fmoe_quantize_groups(torch.zeros(128), 4, torch.zeros(128, dtype=torch.uint8),
                                torch.zeros(2, dtype=torch.int16), torch.zeros(2, dtype=torch.int16))
    # the host tier's layers must hold every routed record
    with pytest.raises(ValueError, match=r"host_layers\[1\]: holds"):
        fm.ExpertCache(d, [torch.zeros(E * d.record_bytes(), dtype=torch.uint8),
                           torch.zeros(E * d.record_bytes() - 1, dtype=torch.uint8)], n_slots=4)
    # a cached layer's descriptor does not need device experts, only the rest
    lw_cached = fm.LayerWeights(d, None, lw.shared, lw.w_router, lw.w_shared_gate, lw.norm_w)
    with pytest.raises(ValueError, match="shared: must be in CUDA device memory"):
        fm.ExpertCache._weights(lw_cached)
