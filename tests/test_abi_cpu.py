"""The C-ABI library loads, exports every entry point declared in
include/cskv.h, and rejects bad arguments on the host before launching
anything (CPU only: no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cskv.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "for")))


@pytest.fixture(scope="module")
def C():
    import compressed_sparse_kv_softmax_b200 as C
    return C


def test_header_declares_the_five_calls():
    d = _declared()
    for n in ("csa_compress", "hca_compress", "indexer_topk", "hybrid_attn_decode",
              "hybrid_attn_prefill"):
        assert n in d


def test_every_declared_symbol_is_exported(C):
    lib = ctypes.CDLL(C.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), f"{name} declared in cskv.h but not exported"


def test_error_strings_and_version(C):
    assert C.error_string(0) == "ok"
    for s in (-1, -2, -3, -4):
        assert C.error_string(s) and C.error_string(s) != "unknown status"
    assert C.version() >= 100


def test_workspace_sizes(C):
    assert C.attn_workspace_size(1, 1, 64, 512, 8192, 128) >= 64 * 513 * 4 * (8192 // 128)
    assert C.indexer_workspace_size(1, 1, 262144, 1024) >= 262144 * 4
    assert C.attn_workspace_size(0, 1, 64, 512, 8192, 128) == 0
    assert C.indexer_workspace_size(1, 1, -1, 8) == 0
    # chunked prefill: room for the dense entries converted once per call into
    # FP16 hi/lo key tiles (128 KB per 64 entries per sequence)
    tiles = 2 * ((8256 + 63) // 64) * 128 * 1024
    assert C.attn_workspace_size(2, 8192, 64, 512, 8256, 128) >= tiles
    assert C.attn_workspace_size(2, 2, 64, 512, 8256, 128) >= tiles


def _fake_cache(ring, cap=256, fmt=1, d_nope=448, d_rope=64, ptr=1 << 20):
    from compressed_sparse_kv_softmax_b200 import CskvCache
    c = CskvCache()
    c.fmt, c.d_nope, c.d_rope, c.ring, c.cap = fmt, d_nope, d_rope, ring, cap
    c.data, c.data_stride = ptr, 448
    c.scale, c.scale_stride = ptr + (1 << 24), 32
    c.rope, c.rope_stride = ptr + (1 << 25), 128
    return c


def test_argument_errors_are_caught_on_the_host(C):
    lib = C.lib
    ERR_ARG, ERR_UNSUP, ERR_WS = C.ERR_ARG, C.ERR_UNSUPPORTED, C.ERR_WORKSPACE
    P = ctypes.c_void_p
    ring, comp = _fake_cache(1), _fake_cache(0, cap=8192)
    q = P(1 << 26)
    ctx = P(1 << 27)
    out = P(1 << 28)
    lse = P(1 << 29)
    ws = P(1 << 30)
    big = 1 << 34
    R = ctypes.byref
    # null query
    assert lib.hybrid_attn_decode(1, ctx, None, 64, 0.04, R(comp), None, 128, None, 0, 8192,
                                  R(ring), None, 128, out, lse, ws, big, None) == ERR_ARG
    # window ring smaller than the window
    small = _fake_cache(1, cap=64)
    assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(comp), None, 128, None, 0, 8192,
                                  R(small), None, 128, out, lse, ws, big, None) == ERR_ARG
    # compressed cache given as a ring
    assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(ring), None, 128, None, 0, 8192,
                                  R(ring), None, 128, out, lse, ws, big, None) == ERR_ARG
    # max_entries beyond the cache
    assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(comp), None, 128, None, 0, 9000,
                                  R(ring), None, 128, out, lse, ws, big, None) == ERR_ARG
    # sparse with k > max_entries
    assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(comp), None, 4, P(1 << 31), 1024, 512,
                                  R(ring), None, 128, out, lse, ws, big, None) == ERR_ARG
    # workspace too small / misaligned
    assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(comp), None, 128, None, 0, 8192,
                                  R(ring), None, 128, out, lse, ws, 16, None) == ERR_WS
    assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(comp), None, 128, None, 0, 8192,
                                  R(ring), None, 128, out, lse, P((1 << 30) + 8), big,
                                  None) == ERR_WS
    # misaligned plane stride
    bad = _fake_cache(0, cap=8192)
    bad.data_stride = 450
    assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(bad), None, 128, None, 0, 8192,
                                  R(ring), None, 128, out, lse, ws, big, None) == ERR_ARG
    # d_nope not a multiple of 64 in the FP8 layout
    odd = _fake_cache(0, cap=8192, d_nope=100)
    assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(odd), None, 128, None, 0, 8192,
                                  R(ring), None, 128, out, lse, ws, big, None) == ERR_UNSUP
    # indexer: k out of range, key cache with rope dims, missing scales
    ik = _fake_cache(0, cap=262144, d_nope=128, d_rope=0)
    ik.data_stride, ik.scale_stride = 128, 8
    args = (1, 1, ctx, q, P(1 << 32), P(1 << 33), 64, 128)
    # (indexer_score / indexer_select check exactly what indexer_topk checks)
    for fn in (lib.indexer_topk, lib.indexer_score, lib.indexer_select):
        assert fn(*args, R(ik), 4, 0, 262144, out, None, ws, big, None) == ERR_ARG
        assert fn(*args, R(ik), 4, 5000, 262144, out, None, ws, big, None) == ERR_ARG
        assert fn(1, 1, ctx, q, None, P(1 << 33), 64, 128, R(ik), 4, 1024, 262144,
                  out, None, ws, big, None) == ERR_ARG
        assert fn(*args, R(ik), 4, 1024, 262145, out, None, ws, big, None) == ERR_ARG
        assert fn(*args, R(comp), 4, 1024, 8192, out, None, ws, big, None) == ERR_ARG
        # more query rows than one call takes (B * Tq > 65,535): refused up front
        assert fn(2, 40000, ctx, q, P(1 << 32), P(1 << 33), 64, 128, R(ik), 4, 1024, 262144,
                  out, None, ws, big, None) == ERR_UNSUP
    # compress: ring too small for the entries requested, pool < stride
    gate = P(1 << 35)
    assert lib.csa_compress(1, ctx, ctx, 100, R(ring), None, None, gate, gate, 8, 4, R(comp),
                            None, None, None) == ERR_ARG
    assert lib.hca_compress(1, ctx, ctx, 1, R(ring), None, gate, gate, 64, 128, R(comp), None,
                            None) == ERR_ARG
    # compress formats: an fp32 indexer ring beside an FP8 KV ring, a per-vector
    # V ring beside a per-64 K ring, a per-vector layout with RoPE dims
    small_ring = _fake_cache(1, cap=16)
    ik_f32 = _fake_cache(1, cap=16, fmt=C.FMT_F32, d_nope=128, d_rope=0)
    ik_f32_out = _fake_cache(0, cap=8192, fmt=C.FMT_F32, d_nope=128, d_rope=0)
    ik_f32.data_stride = ik_f32_out.data_stride = 512
    assert lib.csa_compress(1, ctx, ctx, 1, R(small_ring), None, R(ik_f32), gate, gate, 8, 4,
                            R(comp), None, R(ik_f32_out), None) == ERR_ARG
    v_vec = _fake_cache(1, cap=16, fmt=C.FMT_E4M3_VEC, d_rope=0)
    v_vec_out = _fake_cache(0, cap=8192, fmt=C.FMT_E4M3_VEC, d_rope=0)
    assert lib.csa_compress(1, ctx, ctx, 1, R(small_ring), R(v_vec), None, gate, gate, 8, 4,
                            R(comp), R(v_vec_out), None, None) == ERR_ARG
    vec_rope = _fake_cache(0, cap=8192, fmt=C.FMT_E4M3_VEC)
    assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(vec_rope), None, 128, None, 0, 8192,
                                  R(ring), None, 128, out, lse, ws, big, None) == ERR_UNSUP
    # per-vector indexer keys with a scale stride under 4 bytes
    ik_vec = _fake_cache(0, cap=262144, fmt=C.FMT_E4M3_VEC, d_nope=128, d_rope=0)
    ik_vec.data_stride, ik_vec.scale_stride = 128, 0
    assert lib.indexer_topk(*args, R(ik_vec), 4, 1024, 262144, out, None, ws, big,
                            None) == ERR_ARG
    # paged caches: a paged ring, a block size that is not a power of two or
    # does not divide cap, no blocks; the per-channel compressor's value ring
    # with other channels than the key's, its indexer ring without gates
    paged_ring = _fake_cache(1, cap=16)
    paged_ring.block_table, paged_ring.block_size, paged_ring.num_blocks = 1 << 36, 16, 4
    assert lib.csa_compress(1, ctx, ctx, 1, R(paged_ring), None, None, gate, gate, 8, 4, R(comp),
                            None, None, None) == ERR_ARG
    for bs, nblk in ((48, 512), (16384, 1), (64, 0)):
        pc = _fake_cache(0, cap=8192)
        pc.block_table, pc.block_size, pc.num_blocks = 1 << 36, bs, nblk
        assert lib.hybrid_attn_decode(1, ctx, q, 64, 0.04, R(pc), None, 128, None, 0, 8192,
                                      R(ring), None, 128, out, lse, ws, big, None) == ERR_ARG
    v128 = _fake_cache(1, cap=16, fmt=C.FMT_E4M3_BF16, d_nope=64, d_rope=64)
    v128_out = _fake_cache(0, cap=8192, fmt=C.FMT_E4M3_BF16, d_nope=64, d_rope=64)
    assert lib.csa_compress_channel_gate(1, ctx, ctx, 1, R(small_ring), R(v128), None, gate, gate,
                                         None, None, 8, 4, R(comp), R(v128_out), None,
                                         None) == ERR_ARG
    ik_ring = _fake_cache(1, cap=16, fmt=C.FMT_E4M3_VEC, d_nope=128, d_rope=0)
    ik_out = _fake_cache(0, cap=8192, fmt=C.FMT_E4M3_VEC, d_nope=128, d_rope=0)
    ik_ring.data_stride = ik_out.data_stride = 128
    ik_ring.scale_stride = ik_out.scale_stride = 4
    assert lib.csa_compress_channel_gate(1, ctx, ctx, 1, R(small_ring), None, R(ik_ring), gate,
                                         gate, None, None, 8, 4, R(comp), None, R(ik_out),
                                         None) == ERR_ARG
    # zero-sized work is a no-op success without touching the device
    assert lib.csa_compress(1, ctx, ctx, 0, R(ring), None, None, gate, gate, 8, 4, R(comp),
                            None, None, None) == 0
    assert lib.hybrid_attn_prefill(1, 0, ctx, q, 64, 0.04, R(comp), None, 128, None, 0, 8192,
                                   R(ring), None, 128, out, lse, ws, big, None) == 0


def test_layer_phases_name_the_split_calls(C):
    # CSALayer.select(phase=...) dispatches to the two halves of indexer_topk
    import inspect
    from compressed_sparse_kv_softmax_b200 import layer
    src = inspect.getsource(layer.CSALayer.select)
    for name in ("indexer_topk", "indexer_score", "indexer_select"):
        assert f'"{name}"' in src


def test_prepared_calls_marshal_like_the_plain_calls(C):
    # every call the layers prepare is a library entry point, and a prepared
    # call holds exactly the arguments the plain function passes
    import torch
    for name in C._MARSHAL:
        assert hasattr(C.lib, name), name
    t = [torch.zeros(64, dtype=torch.int64) for _ in range(8)]
    cache = {"fmt": "e4m3vec", "d_nope": 128, "d_rope": 0, "ring": 0, "cap": 16,
             "data": torch.zeros(1, 16, 128, dtype=torch.uint8),
             "scale": torch.zeros(1, 16, 1)}
    ws = torch.zeros(4096, dtype=torch.uint8)
    args = (1, 1, t[0], t[1], t[2], t[3], 64, 128, cache, 4, 8, 16, t[4], t[5], ws, 7)
    call = C.prepare("indexer_score", *args)
    assert call._fn is C.lib.indexer_score
    plain = C._indexer_args(*args)
    for a, b in zip(call._args, plain):
        if isinstance(a, ctypes.c_void_p):
            assert a.value == b.value
        elif isinstance(a, (int, float)):
            assert a == b


def test_header_is_plain_c_and_links(tmp_path):
    # the boundary is a C ABI: the header compiles as C99 with warnings as
    # errors, and a C program links against libcskv.so through it
    import os
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib_dir = os.path.join(root, "compressed_sparse_kv_softmax_b200")
    src = tmp_path / "use.c"
    src.write_text('#include "cskv.h"\n'
                   "#include <stdio.h>\n"
                   "int main(void) {\n"
                   '  printf("%d %s\\n", cskv_version(), cskv_error_string(0));\n'
                   "  return cskv_indexer_workspace_size(1, 1, 1024, 64) == 0;\n"
                   "}\n")
    exe = tmp_path / "use"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(root, "include"), str(src), "-o", str(exe),
                        "-L", lib_dir, "-lcskv", "-Wl,-rpath," + lib_dir],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    assert out.stdout.split()[1] == "ok"

