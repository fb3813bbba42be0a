"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and its host-side logic (sizes, dispatch, validation) holds.

Calls here are either host-only (sizes, dispatch, status strings) or rejected
by argument validation before any CUDA call is made, so they run on a machine
without a GPU.
"""
import ctypes
import functools
import json
import os
import re

import pytest

import weight_only_group_b200 as aq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "aq.h")
GOLDEN = os.path.join(ROOT, "tests", "golden", "storage_arithmetic.json")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if not os.path.exists(aq.LIB_PATH):
        from weight_only_group_b200 import build
        build.build()
    return aq.lib()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(aq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for must in ("aq_quantize", "aq_dequantize", "aq_matmul", "aq_packed_bytes", "aq_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = aq.lib()
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_packed_bytes_match_printed_storage_figures():
    st = json.load(open(GOLDEN))
    # 4.5 bits / weight and 0.5625 bytes / parameter at bits=4, G=64
    assert aq.aq_packed_bytes(64, 64, 64, 4) * 8 / (64 * 64) == st["bits_per_weight_4bit_G64"]["value"]
    assert aq.aq_packed_bytes(4096, 14336, 64, 4) / (4096 * 14336) == st["bytes_per_param_4bit_G64"]["value"]
    # the 70B prediction: N*K = 70,553,706,496 parameters (K = 64 divides it)
    p = st["llama_3_3_70b_prediction"]["params"]
    assert p % 64 == 0
    assert aq.aq_packed_bytes(p // 64, 64, 64, 4) == st["llama_3_3_70b_prediction"]["bytes"]
    r = st["linear_4096x14336_bf16_bytes"]["value"] / aq.aq_packed_bytes(4096, 14336, 64, 4)
    assert abs(r - st["fp16_to_4bit_ratio"]["value"]) <= st["fp16_to_4bit_ratio"]["printed_precision"]


@pytest.mark.parametrize("bits", (2, 3, 4, 8))
@pytest.mark.parametrize("G", (32, 64, 128))
def test_packed_sizes_formula(bits, G):
    N, K = 37, 4 * 128
    assert aq.aq_packed_words(N, K, bits) == N * K * bits // 32
    assert aq.aq_packed_bytes(N, K, G, bits) == N * K * bits // 8 + 4 * N * K // G


def test_packed_sizes_reject_invalid():
    assert aq.aq_packed_bytes(4, 96, 64, 4) == 0      # K % G != 0
    assert aq.aq_packed_bytes(4, 64, 16, 4) == 0      # G unsupported
    assert aq.aq_packed_bytes(4, 64, 64, 5) == 0      # bits unsupported
    assert aq.aq_packed_bytes(0, 64, 64, 4) == 0
    assert aq.aq_packed_words(4, 64, 6) == 0


def test_dispatch_rule():
    # decode shapes -> QMV, prefill shapes -> QMM (the tensor-core kernel)
    for M in range(1, 9):
        assert aq.aq_dispatch(M, 14336, 4096, 64, 4) == aq.AQ_KERNEL_QMV
    assert aq.aq_dispatch(1, 4096, 14336, 64, 4) == aq.AQ_KERNEL_QMV
    assert aq.aq_dispatch(1, 28672, 8192, 32, 3) == aq.AQ_KERNEL_QMV
    for M in (9, 64, 512, 8192):
        assert aq.aq_dispatch(M, 14336, 4096, 64, 4) == aq.AQ_KERNEL_QMM
    # many tokens over a long K: the decode kernel in token chunks (staged x of a
    # launch within 120 KB: 4 tokens at K = 14336), not the prefill kernel
    for M in range(1, 9):
        assert aq.aq_dispatch(M, 4096, 14336, 64, 4) == aq.AQ_KERNEL_QMV
    # 3-bit codes have no tensor-core decode; beyond its CUDA-core kernel's shared memory: QMM
    assert aq.aq_dispatch(8, 200, 14336, 32, 3) == aq.AQ_KERNEL_QMM
    # invalid shapes
    assert aq.aq_dispatch(0, 4096, 4096, 64, 4) == -1
    assert aq.aq_dispatch(1, 4096, 4000, 64, 4) == -1
    assert aq.aq_dispatch(1, 4096, 4096, 64, 7) == -1


def test_status_strings():
    for s in range(6):
        assert aq.aq_status_string(s)
    assert "unknown" in aq.aq_status_string(99)


# Fake device pointers: every call below is rejected by host-side validation
# before any CUDA call, so nothing is dereferenced.
A = 0x10000  # 16-byte aligned
U = 0x10004  # misaligned


def _q(w=A, N=4, K=64, G=64, bits=4, p=A, s=A, b=A, fn="aq_quantize"):
    return getattr(aq.lib(), fn)(w, N, K, G, bits, p, s, b, None)


@pytest.mark.parametrize("fn", ("aq_quantize", "aq_quantize_mse"))
def test_quantize_validation(fn):
    _q = functools.partial(globals()["_q"], fn=fn)
    assert _q(bits=5) == aq.AQ_ERR_UNSUPPORTED
    assert _q(G=16) == aq.AQ_ERR_UNSUPPORTED
    assert _q(K=96) == aq.AQ_ERR_INVALID_ARG
    assert _q(N=0) == aq.AQ_ERR_INVALID_ARG
    assert _q(K=-64) == aq.AQ_ERR_INVALID_ARG
    assert _q(w=0) == aq.AQ_ERR_INVALID_ARG
    assert _q(p=0) == aq.AQ_ERR_INVALID_ARG
    assert _q(w=U) == aq.AQ_ERR_ALIGNMENT
    assert _q(s=U) == aq.AQ_ERR_ALIGNMENT


def test_matmul_validation():
    L = aq.lib()
    call = lambda k=0, x=A, M=1, K=64, N=8, G=64, bits=4, y=A: L.aq_matmul_with(k, x, M, K, A, A, A, N, G, bits, y,
                                                                                 None)
    assert call(bits=1) == aq.AQ_ERR_UNSUPPORTED
    assert call(M=0) == aq.AQ_ERR_INVALID_ARG
    assert call(x=0) == aq.AQ_ERR_INVALID_ARG
    assert call(y=U) == aq.AQ_ERR_ALIGNMENT
    assert call(k=7) == aq.AQ_ERR_INVALID_ARG
    # QMV forced beyond its range
    assert call(k=aq.AQ_KERNEL_QMV, M=9) == aq.AQ_ERR_UNSUPPORTED
    # QMM needs a 16-byte packed row pitch: K*bits % 128 == 0 (K=96, 3 bits: 288 bits)
    assert call(k=aq.AQ_KERNEL_QMM, M=64, K=96, G=32, bits=3) == aq.AQ_ERR_UNSUPPORTED
    assert L.aq_dequantize(A, A, A, 4, 64, 64, 4, U, None) == aq.AQ_ERR_ALIGNMENT
    assert L.aq_dequantize_f32(A, A, A, 4, 64, 64, 9, A, None) == aq.AQ_ERR_UNSUPPORTED


def test_matmul_ex_flags():
    L = aq.lib()
    call = lambda flags: L.aq_matmul_ex(A, 1, 64, A, A, A, 8, 64, 4, A, flags, None)
    assert call(2) == aq.AQ_ERR_INVALID_ARG          # unknown flag bit
    assert call(1 << 31) == aq.AQ_ERR_INVALID_ARG
    assert L.aq_matmul_ex(A, 0, 64, A, A, A, 8, 64, 4, A, aq.AQ_MATMUL_OVERLAP_PREVIOUS, None) == aq.AQ_ERR_INVALID_ARG


def test_matmul_sequence_validation():
    """Argument checks of aq_matmul_sequence, all before any device work."""
    L = aq.lib()
    D = aq._MatmulDesc

    def call(n=2, M=1, G=64, bits=4, flags=0, **kw):
        f = dict(x_bf16=A, packed=A, scales=A, biases=A, y_bf16=A, N=1024, K=2048)
        f.update(kw)
        arr = (D * 4)(*[D(**f) for _ in range(4)])
        return L.aq_matmul_sequence(arr, n, M, G, bits, flags, None)

    assert L.aq_matmul_sequence(None, 1, 1, 64, 4, 0, None) == aq.AQ_ERR_INVALID_ARG
    assert call(n=0) == aq.AQ_ERR_INVALID_ARG
    assert call(n=5) == aq.AQ_ERR_INVALID_ARG
    assert call(M=0) == aq.AQ_ERR_INVALID_ARG
    assert call(flags=2) == aq.AQ_ERR_INVALID_ARG
    assert call(x_bf16=0) == aq.AQ_ERR_INVALID_ARG
    assert call(M=9) == aq.AQ_ERR_UNSUPPORTED
    assert call(bits=3) == aq.AQ_ERR_UNSUPPORTED
    assert call(G=16) == aq.AQ_ERR_UNSUPPORTED
    assert call(y_bf16=U) == aq.AQ_ERR_ALIGNMENT
    assert call(K=96) == aq.AQ_ERR_INVALID_ARG      # K not a multiple of G
    assert call(K=64 * 4) == aq.AQ_ERR_UNSUPPORTED  # K not a multiple of 8 G
    assert call(N=8) == aq.AQ_ERR_UNSUPPORTED       # fewer than 16 rows


def test_embedding_validation():
    L = aq.lib()
    call = lambda ids=A, T=4, V=100, D=64, G=64, bits=4, out=A: L.aq_embedding(ids, T, A, A, A, V, D, G, bits, out, None)
    assert call(T=0) == aq.AQ_ERR_INVALID_ARG
    assert call(V=0) == aq.AQ_ERR_INVALID_ARG
    assert call(D=96) == aq.AQ_ERR_INVALID_ARG          # D % G != 0
    assert call(G=16) == aq.AQ_ERR_UNSUPPORTED
    assert call(bits=6) == aq.AQ_ERR_UNSUPPORTED
    assert call(ids=0) == aq.AQ_ERR_INVALID_ARG
    assert call(ids=A + 2) == aq.AQ_ERR_ALIGNMENT         # ids need 4-byte alignment
    assert call(out=U) == aq.AQ_ERR_ALIGNMENT


def test_gather_matmul_validation():
    L = aq.lib()
    def call(x=A, T=2, K=4096, E=8, N=1024, G=64, bits=4, experts=A, y=A):
        return L.aq_gather_matmul(x, T, K, A, A, A, E, N, G, bits, experts, y, None)
    assert call(T=0) == aq.AQ_ERR_INVALID_ARG
    assert call(E=0) == aq.AQ_ERR_INVALID_ARG
    assert call(K=4000) == aq.AQ_ERR_INVALID_ARG         # K % G != 0
    assert call(experts=0) == aq.AQ_ERR_INVALID_ARG
    assert call(experts=A + 2) == aq.AQ_ERR_ALIGNMENT
    assert call(y=U) == aq.AQ_ERR_ALIGNMENT
    assert call(bits=3) == aq.AQ_ERR_UNSUPPORTED          # the gather path is the tensor-core QMV (2/4/8-bit)
    assert call(K=4096 + 64) == aq.AQ_ERR_UNSUPPORTED     # K not a multiple of 8*G
    assert call(N=8) == aq.AQ_ERR_UNSUPPORTED             # fewer than 16 rows
    assert call(E=1 << 20, N=4096) == aq.AQ_ERR_INVALID_ARG  # E*N >= 2^31


def test_gather_matmul_grouped_validation():
    L = aq.lib()
    def call(x=A, T=64, K=4096, E=8, N=1024, G=64, bits=4, experts=A, y=A):
        return L.aq_gather_matmul_grouped(x, T, K, A, A, A, E, N, G, bits, experts, y, None)
    assert call(T=0) == aq.AQ_ERR_INVALID_ARG
    assert call(E=0) == aq.AQ_ERR_INVALID_ARG
    assert call(E=20000, N=64) == aq.AQ_ERR_INVALID_ARG    # more experts than the routing CTA takes
    assert call(K=4000) == aq.AQ_ERR_INVALID_ARG           # K % G != 0
    assert call(experts=A + 2) == aq.AQ_ERR_ALIGNMENT
    assert call(x=U) == aq.AQ_ERR_ALIGNMENT
    assert call(N=1028) == aq.AQ_ERR_UNSUPPORTED           # segments of y must stay 16-byte aligned
    assert call(bits=5) == aq.AQ_ERR_UNSUPPORTED


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        aq.aq_quantize(torch.zeros(4, 64), 64, 4)


def test_workspace_size_rule():
    assert aq.aq_matmul_workspace_bytes(1, 4096, 4096, 64, 4) == 0          # QMV: none
    need = aq.aq_matmul_workspace_bytes(512, 4096, 4096, 64, 4)            # QMM: fp16 x + row scales
    assert need >= 512 * 4096 * 2 + 512 * 4
    assert aq.aq_matmul_workspace_bytes(512, 4096, 4000, 64, 4) == 0       # rejected shape


def test_workspace_size_k_split():
    """A CTA-pair shape (M > 128, N % 8 == 0) whose T tiles of 256 x 256 fill at
    most half of 74 pairs cuts each tile's K range into ks = min(74 // T, 4,
    K blocks // 32) parts (K blocks of 64, 128 for 3-bit codes; split when
    ks >= 2).  Its workspace then adds one uint32 arrival counter per (tile, CTA,
    dequant warp), 256-byte padded, and ks*T*2*128*256 fp32 partial sums to the
    activations' part; other shapes need the activations' part alone."""
    def base(M, K):
        r = lambda b: (b + 255) // 256 * 256
        return r(M * K * 2) + r(M * 4)
    tile2 = 2 * 128 * 256 * 4
    ws = aq.aq_matmul_workspace_bytes
    assert ws(512, 4096, 14336, 64, 4) == base(512, 14336) + 3072 + 2 * 32 * tile2   # 32 tiles, 2 parts
    assert ws(257, 776, 8192, 128, 2) == base(257, 8192) + 768 + 4 * 8 * tile2      # 8 tiles, 4 parts (2-bit)
    assert ws(129, 256, 6144, 32, 8) == base(129, 6144) + 256 + 3 * 1 * tile2       # 1 tile, 96 blocks: 3 parts
    assert ws(256, 9472, 4096, 64, 4) == base(256, 4096) + 3584 + 2 * 37 * tile2     # 37 tiles: 74 items
    assert ws(160, 264, 6144, 32, 3) == base(160, 6144)          # 3-bit: 48 blocks of 128, too few for two parts
    assert ws(256, 9728, 4096, 64, 4) == base(256, 4096)         # 38 tiles: more than half the pairs
    assert ws(2048, 4096, 14336, 64, 4) == base(2048, 14336)     # 128 tiles
    assert ws(700, 300, 2048, 64, 4) == base(700, 2048)          # 32 K blocks
    assert ws(128, 4096, 14336, 64, 4) == base(128, 14336)       # single-CTA kernel


def test_workspace_validation():
    L = aq.lib()
    # a QMM shape with no workspace -> invalid argument, before any CUDA call
    assert L.aq_matmul_ws(A, 512, 4096, A, A, A, 64, 64, 4, A, None, 0, None) == aq.AQ_ERR_INVALID_ARG
    assert L.aq_matmul_ws(A, 512, 4096, A, A, A, 64, 64, 4, A, A, 16, None) == aq.AQ_ERR_INVALID_ARG
    assert L.aq_matmul_ws(A, 512, 4096, A, A, A, 64, 64, 4, A, U, 1 << 30, None) == aq.AQ_ERR_ALIGNMENT


def test_mxfp4_validation():
    L = aq.lib()
    assert aq.aq_mxfp4_packed_bytes(4096, 4096) == 4096 * 4096 // 2 + 4096 * 4096 // 32
    assert aq.aq_mxfp4_packed_bytes(4, 48) == 0
    assert L.aq_mxfp4_quantize(A, 4, 48, A, A, None) == aq.AQ_ERR_INVALID_ARG      # K % 32
    assert L.aq_mxfp4_quantize(A, 0, 64, A, A, None) == aq.AQ_ERR_INVALID_ARG
    assert L.aq_mxfp4_quantize(0, 4, 64, A, A, None) == aq.AQ_ERR_INVALID_ARG
    assert L.aq_mxfp4_quantize(U, 4, 64, A, A, None) == aq.AQ_ERR_ALIGNMENT
    assert L.aq_mxfp4_dequantize(A, U, 4, 64, A, None) == aq.AQ_ERR_ALIGNMENT
    assert L.aq_mxfp4_dequantize_f32(A, A, 4, 40, A, None) == aq.AQ_ERR_INVALID_ARG
    mm = lambda M=1, K=512, N=16, flags=0, x=A: L.aq_mxfp4_matmul(x, M, K, A, A, N, A, flags, None)
    assert mm(K=256) == aq.AQ_ERR_UNSUPPORTED          # the decode kernel needs K % 512 == 0
    assert mm(M=9) not in (aq.AQ_ERR_INVALID_ARG, aq.AQ_ERR_UNSUPPORTED, aq.AQ_ERR_ALIGNMENT)  # prefill: valid (needs a device)
    assert mm(N=8) == aq.AQ_ERR_UNSUPPORTED            # at least one 16-row tile
    assert mm(flags=2) == aq.AQ_ERR_INVALID_ARG
    assert mm(x=U) == aq.AQ_ERR_ALIGNMENT
    assert mm(M=0) == aq.AQ_ERR_INVALID_ARG


def test_nvfp4_validation():
    L = aq.lib()
    assert aq.aq_nvfp4_packed_bytes(4096, 4096) == 4096 * 4096 // 2 + 4096 * 4096 // 16 + 4
    assert L.aq_nvfp4_quantize(A, 4, 48, A, A, A, None) == aq.AQ_ERR_INVALID_ARG     # K % 32
    assert L.aq_nvfp4_quantize(A, 4, 64, A, A, 0, None) == aq.AQ_ERR_INVALID_ARG     # no tensor scale
    assert L.aq_nvfp4_quantize(A, 4, 64, A, A, A + 2, None) == aq.AQ_ERR_ALIGNMENT
    assert L.aq_nvfp4_dequantize(A, U, A, 4, 64, A, None) == aq.AQ_ERR_ALIGNMENT
    mm = lambda M=1, K=512, N=16, flags=0: L.aq_nvfp4_matmul(A, M, K, A, A, A, N, A, flags, None)
    assert mm(M=9) not in (aq.AQ_ERR_INVALID_ARG, aq.AQ_ERR_UNSUPPORTED, aq.AQ_ERR_ALIGNMENT)  # prefill: valid (needs a device)
    assert mm(K=208) == aq.AQ_ERR_INVALID_ARG      # K % 32 != 0
    assert mm(K=288) == aq.AQ_ERR_UNSUPPORTED      # the decode kernel needs K % 256 == 0
    assert mm(N=8) == aq.AQ_ERR_UNSUPPORTED
    assert mm(flags=4) == aq.AQ_ERR_INVALID_ARG


def test_mxfp8_validation():
    L = aq.lib()
    assert aq.aq_mxfp8_packed_bytes(4096, 4096) == 4096 * 4096 + 4096 * 4096 // 32
    assert L.aq_mxfp8_quantize(A, 4, 48, A, A, None) == aq.AQ_ERR_INVALID_ARG
    assert L.aq_mxfp8_quantize(U, 4, 64, A, A, None) == aq.AQ_ERR_ALIGNMENT
    assert L.aq_mxfp8_dequantize_f32(A, A, 4, 40, A, None) == aq.AQ_ERR_INVALID_ARG
    mm = lambda M=1, K=512, N=16, flags=0: L.aq_mxfp8_matmul(A, M, K, A, A, N, A, flags, None)
    assert mm(K=256) == aq.AQ_ERR_UNSUPPORTED
    assert mm(M=9) not in (aq.AQ_ERR_INVALID_ARG, aq.AQ_ERR_UNSUPPORTED, aq.AQ_ERR_ALIGNMENT)  # prefill: valid (needs a device)
    assert mm(N=8) == aq.AQ_ERR_UNSUPPORTED
    assert mm(flags=8) == aq.AQ_ERR_INVALID_ARG
