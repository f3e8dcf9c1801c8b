"""The C-ABI library loads, exports every symbol the header declares, and
rejects invalid arguments on the host (no GPU needed, no kernel launched)."""
import ctypes
import os
import re

import pytest

from sparse_attention_logits_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    path = _build.build_library()
    return ctypes.CDLL(path)


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"DSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"csa_compress", "dsa_indexer_logits", "dsa_topk", "dsa_sparse_mla", "dsa_get_device_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_only_the_abi_is_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB_PATH], capture_output=True, text=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.strip()}
    declared = set(_declared())
    extra = {s for s in syms if not (s in declared or s.startswith("_"))}
    assert not extra, f"exports not declared in include/: {sorted(extra)[:10]}"


def test_version(lib):
    assert lib.dsa_version() >= 100


def _err(lib):
    lib.dsa_last_error.restype = ctypes.c_char_p
    return lib.dsa_last_error().decode()


def test_invalid_arguments_rejected_before_launch(lib):
    vp = ctypes.c_void_p
    fake = vp(0x1000)      # never dereferenced: validation fails first
    # top-k with k = 0
    lib.dsa_topk.argtypes = [vp, ctypes.c_int64, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp,
                             ctypes.c_size_t, vp]
    assert lib.dsa_topk(fake, 100, fake, 4, 100, 0, fake, None, 0, None) == 1
    assert "k must be" in _err(lib)
    # ld < ctx_len
    assert lib.dsa_topk(fake, 10, fake, 4, 100, 5, fake, None, 0, None) == 1
    # compress: len not a multiple of m
    lib.csa_compress.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
    assert lib.csa_compress(fake, 1, 2, 10, 576, 4, vp(0x100000), None) == 1
    # compress: unsupported dtype (fp8)
    assert lib.csa_compress(fake, 2, 2, 8, 576, 4, vp(0x100000), None) == 2
    # compress: overlapping buffers
    assert lib.csa_compress(vp(0x10000), 1, 1, 8, 64, 4, vp(0x10000 + 64), None) == 1
    # indexer: fp8 keys without scales
    lib.dsa_indexer_logits.argtypes = [vp, ctypes.c_int, vp, vp, ctypes.c_int, vp, vp, vp, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int64, vp]
    assert lib.dsa_indexer_logits(fake, 1, fake, fake, 2, None, fake, fake, 4, 4, 128, 64, 128, fake, 128, None) == 1
    # indexer: unsupported head dim
    assert lib.dsa_indexer_logits(fake, 1, fake, fake, 1, None, fake, fake, 4, 4, 128, 64, 96, fake, 128, None) == 2
    # sparse MLA: null output
    lib.dsa_sparse_mla.argtypes = [vp, vp, ctypes.c_int, vp, ctypes.c_int, ctypes.c_int, vp, vp, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_float, vp, vp, vp, ctypes.c_size_t, vp]
    assert lib.dsa_sparse_mla(fake, fake, 1, None, 0, 0, fake, fake, 2048, 4, 4, 4096, 128, 576, 512, 0.04, None,
                              fake, None, 0, None) == 1
    # sparse MLA: unbuilt head geometry
    assert lib.dsa_sparse_mla(fake, fake, 1, None, 0, 0, fake, fake, 2048, 4, 4, 4096, 100, 576, 512, 0.04, fake,
                              fake, None, 0, None) == 2
    # paged cache without a page count
    assert lib.dsa_sparse_mla(fake, fake, 1, fake, 64, 0, fake, fake, 2048, 4, 4, 4096, 128, 576, 512, 0.04, fake,
                              fake, None, 0, None) == 1
    # zero rows is a no-op success without touching the device
    assert lib.dsa_topk(fake, 100, fake, 0, 100, 5, fake, None, 0, None) == 0
    # indexer: fp4 keys without scales; fp4 keys with a head geometry no kernel is built for
    assert lib.dsa_indexer_logits(fake, 1, fake, fake, 3, None, fake, fake, 4, 4, 128, 64, 128, fake, 128, None) == 1
    assert lib.dsa_indexer_logits(fake, 1, fake, fake, 3, fake, fake, fake, 4, 4, 128, 64, 64, fake, 128, None) == 2
    assert "fp4" in _err(lib)


def test_v4_attention_arguments_rejected_before_launch(lib):
    vp, ci = ctypes.c_void_p, ctypes.c_int
    fake = vp(0x1000)      # never dereferenced: validation fails first
    lib.csa_core_attention.argtypes = [vp, vp, ci, vp, ci, ci, vp, vp, ci, ci, ci, ci, vp, vp, ci, ci, ci, ci, ci,
                                       ci, ctypes.c_float, vp, vp, vp, ctypes.c_size_t, vp]

    def csa(idx, k, kv_win, win_pos, win_len, window, n_heads=128, n_sink=0):
        return lib.csa_core_attention(fake, fake, 1, None, 0, 0, fake, idx, k, 4, 4, 1024, kv_win, win_pos, win_len,
                                      window, n_sink, n_heads, 576, 512, 0.04, fake, fake, None, 0, None)
    assert csa(fake, 64, fake, fake, 4096, -1) == 1                  # negative window
    assert csa(fake, 64, fake, fake, 4096, 128, n_sink=-1) == 1      # negative sink
    assert csa(fake, 64, None, fake, 4096, 0, n_sink=4) == 1         # sink without its cache
    assert csa(fake, 64, fake, None, 4096, 0, n_sink=4) == 1         # sink without positions
    assert csa(fake, 64, fake, fake, 16, 8, n_sink=17) == 1          # more sink rows than the raw cache holds
    assert csa(fake, 64, None, fake, 4096, 128) == 1                 # window without its cache
    assert csa(fake, 64, fake, None, 4096, 128) == 1                 # window without positions
    assert csa(None, 0, fake, fake, 4096, 0) == 1                    # no slot at all
    assert csa(None, 64, fake, fake, 4096, 128) == 1                 # selected slots without an index list
    assert csa(fake, 64, fake, fake, 4096, 128, n_heads=100) == 2    # no kernel for this geometry
    lib.hca_attention.argtypes = [vp, vp, ci, vp, vp, ci, ci, ci, ci, ci, ci, ctypes.c_float, vp, vp, vp,
                                  ctypes.c_size_t, vp]
    assert lib.hca_attention(fake, fake, 1, fake, None, 4, 4, 8192, 128, 576, 512, 0.04, fake, fake, None, 0,
                             None) == 1                              # no row_last
    assert lib.hca_attention(fake, fake, 1, fake, fake, 4, 4, 8192, 100, 576, 512, 0.04, fake, fake, None, 0,
                             None) == 2                              # no kernel for this geometry
    assert lib.hca_attention(fake, fake, 1, fake, fake, 0, 4, 8192, 128, 576, 512, 0.04, fake, fake, None, 0,
                             None) == 0                              # zero rows: nothing to do


def test_indexer_prepare_arguments_rejected_before_launch(lib):
    vp, ci, cf, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64, ctypes.c_size_t
    fake = vp(0x1000)      # never dereferenced: validation fails first
    lib.dsa_indexer_prepare.argtypes = [vp, vp, cf, vp, vp, vp, vp, vp, vp, ci, ci, vp, vp, ci, ci, ci, ci, ci, vp,
                                        vp, vp, ci, vp, i64, vp, sz, vp]

    def prep(tokens=64, d_c=1536, d_model=7168, head_dim=128, d_rope=64, tables=True, fmt=2, scale=True,
             c_q=fake, eps=1e-6, slot=fake):
        tab = fake if tables else None
        return lib.dsa_indexer_prepare(c_q, fake, eps, fake, fake, fake, fake, tab, tab, 4096, d_rope, fake, slot,
                                       tokens, d_c, d_model, 64, head_dim, fake, fake, fake, fmt,
                                       fake if scale else None, 1 << 20, fake, 1 << 30, None)
    assert prep(tokens=0) == 0                       # nothing to do
    assert prep(head_dim=64) == 2                    # keys are 128-dim
    assert prep(d_rope=63) == 1                      # odd rotary part
    assert prep(d_rope=130) == 1                     # rotary part longer than the head
    assert prep(tables=False) == 1                   # rotary part without tables
    assert prep(fmt=1, scale=True) == 1              # bf16 cache with a scale array
    assert prep(fmt=2, scale=False) == 1             # fp8 cache without one
    assert prep(fmt=0, scale=False) == 2             # fp32 cache: no such format
    assert prep(d_c=1000) == 2                       # reduction not a multiple of 64
    assert prep(c_q=vp(0x1002)) == 1                 # misaligned activation
    assert prep(eps=-1.0) == 1
    assert prep(slot=None) == 1
    lib.dsa_indexer_key_append.argtypes = [vp, ci, vp, vp, ci, ci, vp, vp, ci, ci, vp, ci, vp, i64, vp]

    def app(k=fake, k_dt=1, n=8, head_dim=128, fmt=3, scale=True):
        return lib.dsa_indexer_key_append(k, k_dt, None, None, 0, 0, None, fake, n, head_dim, fake, fmt,
                                          fake if scale else None, 1 << 20, None)
    assert app(n=0) == 0
    assert app(k_dt=2) == 2                          # fp8 input keys
    assert app(head_dim=64) == 2
    assert app(k=vp(0x1004)) == 1
    assert app(scale=False) == 1                     # fp4 cache without scales


def test_indexer_prepare_workspace_sizes(lib):
    # no device here: the size is taken for a 1024-SM GPU (the most splits).
    # Layout: fp32 partials of 128 key + 64 weight columns for 128 token rows
    # per split and token tile | the scaled latent, [tokens, d_c] bf16 |
    # 1/RMS, [tokens] fp32, each part starting on a 256-byte boundary.
    lib.dsa_indexer_prepare_workspace_size.restype = ctypes.c_size_t
    lib.dsa_indexer_prepare_workspace_size.argtypes = [ctypes.c_int] * 4

    def up(x):
        return (x + 255) // 256 * 256

    def size(T, d_c, splits):
        tiles = (T + 127) // 128
        part = splits * tiles * 128 * 192 * 4
        inv = up(up(part) + T * d_c * 2)
        return inv + T * 4

    # 64 tokens: one token tile, the 112-chunk d_model reduction split 5 ways
    # (about the 24 chunks of a query tile)
    assert lib.dsa_indexer_prepare_workspace_size(64, 64, 1536, 7168) == size(64, 1536, 5) == 688384
    # 16384 tokens: 256-wide query tiles fill the GPU, no split
    assert lib.dsa_indexer_prepare_workspace_size(16384, 64, 1536, 7168) == size(16384, 1536, 1) == 62980096
    assert lib.dsa_indexer_prepare_workspace_size(0, 64, 1536, 7168) == 0


def test_key_cache_format_inference():
    torch = pytest.importorskip("torch")
    dsa = pytest.importorskip("sparse_attention_logits_b200")
    assert dsa._key_cache_fmt(torch.zeros(10, 128, dtype=torch.bfloat16)) == (dsa.DSA_BF16, 10)
    assert dsa._key_cache_fmt(torch.zeros(2, 5, 128, dtype=torch.uint8)) == (dsa.DSA_FP8_E4M3, 10)
    assert dsa._key_cache_fmt(torch.zeros(2, 5, 64, dtype=torch.uint8)) == (dsa.DSA_FP4_E2M1, 10)
    with pytest.raises(TypeError):
        dsa._key_cache_fmt(torch.zeros(10, 128, dtype=torch.float32))


def test_sparse_mla_workspace_size_without_device_bounds_every_gpu(lib):
    # No device here: the size is taken for a 1024-SM GPU.  The split count
    # grows with the SM count (up to one split per 64 selected keys), so this
    # must be at least what a 148-SM B200 asks for.  A (row, split) pair holds
    # a bf16 partial of 128 heads x 512 dims and an fp32 lse per head.
    lib.dsa_sparse_mla_workspace_size.restype = ctypes.c_size_t
    lib.dsa_sparse_mla_workspace_size.argtypes = [ctypes.c_int] * 6
    pair = 128 * (512 * 2 + 4)

    def b200_size(rows, k):                       # the split rule on 148 SMs (74 CTA pairs)
        s = 1 if rows >= 74 else 74 // rows
        s = max(1, min(s, (k + 63) // 64))
        return 0 if s == 1 else rows * s * pair

    for rows, k in ((2, 2048), (4, 1152), (32, 2048), (64, 2048), (1, 64)):
        got = lib.dsa_sparse_mla_workspace_size(rows, k, 128, 576, 512, 1)
        assert got >= b200_size(rows, k), (rows, k, got)
    assert lib.dsa_sparse_mla_workspace_size(2, 2048, 128, 576, 512, 1) == 2 * 32 * pair   # one split per 64 keys
    assert lib.dsa_sparse_mla_workspace_size(0, 2048, 128, 576, 512, 1) == 0
