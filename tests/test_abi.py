"""The C-ABI library loads without a GPU, exports every entry point that
include/pkv.h declares, and rejects bad arguments on the host before any
launch (none of these calls reaches the GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(pkv_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "pkv_build", os.path.join(ROOT, "paged_kv_attention_37_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("pkv_kv_append", "pkv_paged_attn_decode", "pkv_paged_attn_chunked_prefill",
              "pkv_split_k_combine", "pkv_decode_workspace_bytes", "pkv_status_string",
              "pkv_device_error_flags"):
        assert n in names, n


def test_library_exports_every_declared_symbol(lib):
    path = lib._name
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (pkv_\w+)$", out, flags=re.M))
    declared = set(declared_functions())
    assert declared <= exported, declared - exported
    # nothing but the declared ABI is exported under the pkv_ prefix
    assert exported <= declared, exported - declared
    for name in declared:
        assert getattr(lib, name) is not None


class PoolDesc(ctypes.Structure):
    _fields_ = [("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


def test_status_strings(lib):
    lib.pkv_status_string.restype = ctypes.c_char_p
    for st in range(0, -9, -1):
        s = lib.pkv_status_string(st).decode()
        assert s and s != "unknown status"
    assert lib.pkv_status_string(-99).decode() == "unknown status"


def test_workspace_size(lib):
    lib.pkv_decode_workspace_bytes.restype = ctypes.c_size_t
    f = lib.pkv_decode_workspace_bytes
    # no split: header + num_splits + one partial per (request, head)
    small = f(4, 32, 128, 4096, -1)
    assert small >= 256 + 4 * 4 + 4 * 32 * 4 + 4 * 32 * 128 * 4
    # auto: sized for the smallest automatic partition (256 tokens)
    auto = f(4, 32, 64, 131072, 0)
    assert auto >= 4 * 32 * 512 * 64 * 4
    assert f(4, 32, 64, 131072, 4096) < auto
    assert f(-1, 32, 64, 10, 0) == 0


def test_workspace_holds_the_merge_tree(lib):
    # Under the automatic split a (request, KV head) group is cut into at most
    # n = ceil(L / 128) + 1 pieces; the pieces and every inner level of their
    # merge tree (fan-in 8 at d = 128, 16 at d = 64: each level a ceiling
    # division of the one below, until one node is left) need partial slots.
    lib.pkv_decode_workspace_bytes.restype = ctypes.c_size_t
    f = lib.pkv_decode_workspace_bytes

    def slots(n, fan):
        levels = [n]
        while levels[-1] > 1:
            levels.append(-(-levels[-1] // fan))
        return sum(levels[:-1]) if len(levels) > 1 else 1

    B, Hq = 3, 32
    prev = 0
    for d, fan in ((128, 8), (64, 16)):
        for L in (1, 100, 1000, 1024, 1025, 8192, 8193, 65536, 131072):
            n = -(-L // 128) + 1
            got = f(B, Hq, d, L, 0)
            assert got >= B * Hq * slots(n, fan) * (d + 1) * 4, (d, L)
            if d == 128:
                assert got >= prev  # grows with the longest context
                prev = got
    # a tree of more than one level holds more than its pieces alone
    assert slots(9, 8) == 9 + 2 and slots(65, 8) == 65 + 9 + 2 and slots(8, 8) == 8


def test_host_validation_without_gpu(lib):
    good = PoolDesc(64, 16, 8, 128)
    dummy = ctypes.c_void_p(16)
    lib.pkv_kv_append.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int32] + \
        [ctypes.c_void_p] * 2 + [PoolDesc, ctypes.c_void_p]
    # unsupported head_dim / page_size
    assert lib.pkv_kv_append(dummy, dummy, dummy, 4, dummy, dummy, PoolDesc(64, 16, 8, 96), None) == -3
    assert lib.pkv_kv_append(dummy, dummy, dummy, 4, dummy, dummy, PoolDesc(64, 8, 8, 128), None) == -3
    # negative token count; empty batch is a no-op
    assert lib.pkv_kv_append(dummy, dummy, dummy, -1, dummy, dummy, good, None) == -2
    assert lib.pkv_kv_append(None, None, None, 0, None, None, good, None) == 0
    # null pointer, misaligned pointer
    assert lib.pkv_kv_append(None, dummy, dummy, 4, dummy, dummy, good, None) == -1
    assert lib.pkv_kv_append(ctypes.c_void_p(18), dummy, dummy, 4, dummy, dummy, good, None) == -4

    P, I32 = ctypes.c_void_p, ctypes.c_int32
    lib.pkv_paged_attn_decode.argtypes = [P, I32, I32, P, P, PoolDesc, P, I32, P, ctypes.c_float,
                                          I32, P, ctypes.c_size_t, P, P, P]
    dec = lib.pkv_paged_attn_decode
    # Hq not a multiple of Hkv; group size 16 unsupported
    assert dec(dummy, 4, 12, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, dummy, 1 << 20, dummy, None, None) == -2
    assert dec(dummy, 4, 128, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, dummy, 1 << 20, dummy, None, None) == -3
    # partition not a multiple of 32
    assert dec(dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 100, dummy, 1 << 20, dummy, None, None) == -2
    # workspace too small
    ws = ctypes.c_void_p(4096)
    assert dec(dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, ws, 64, dummy, None, None) == -5
    # non-finite scale
    assert dec(dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, float("nan"), 0, ws, 1 << 20, dummy, None, None) == -2

    # the scratch-free entry point runs the same checks before touching its scratch
    lib.pkv_paged_attn_decode_static.argtypes = [P, I32, I32, P, P, PoolDesc, P, I32, P, ctypes.c_float,
                                                 I32, P, P, P]
    sdec = lib.pkv_paged_attn_decode_static
    assert sdec(dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 33, dummy, None, None) == -2
    assert sdec(dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 65536 + 32, dummy, None, None) == -2
    assert sdec(dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, float("inf"), 0, dummy, None, None) == -2
    assert sdec(dummy, 4, 12, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, dummy, None, None) == -2
    assert sdec(None, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, dummy, None, None) == -1
    # a partition below -1 is not one of the documented values
    assert dec(dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, -5, ws, 1 << 20, dummy, None, None) == -2

    lib.pkv_paged_attn_decode_flags.argtypes = [P, I32, I32, P, P, PoolDesc, P, I32, P, ctypes.c_float,
                                                I32, P, ctypes.c_size_t, P, P, ctypes.c_uint32, P]
    decf = lib.pkv_paged_attn_decode_flags
    assert decf(dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, ws, 1 << 20, dummy, None, 2, None) == -2
    assert decf(dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, ws, 64, dummy, None, 1, None) == -5

    lib.pkv_paged_attn_decode_append.argtypes = [P, P, P, I32, I32, P, P, PoolDesc, P, I32, P, ctypes.c_float,
                                                 I32, P, ctypes.c_size_t, P, P, ctypes.c_uint32, P]
    deca = lib.pkv_paged_attn_decode_append
    # unknown option bit; new rows missing; new rows misaligned; workspace too small
    assert deca(dummy, dummy, dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, ws, 1 << 20, dummy, None,
                2, None) == -2
    assert deca(dummy, None, dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, ws, 1 << 20, dummy, None,
                0, None) == -1
    assert deca(dummy, dummy, ctypes.c_void_p(24), 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, ws,
                1 << 20, dummy, None, 0, None) == -4
    assert deca(dummy, dummy, dummy, 4, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, ws, 64, dummy, None, 1,
                None) == -5
    # an empty batch is a valid call that launches nothing
    assert deca(None, None, None, 0, 32, dummy, dummy, good, dummy, 8, dummy, 0.1, 0, None, 0, None, None, 0,
                None) == 0

    lib.pkv_paged_attn_verify.argtypes = [P, P, I32, I32, I32, I32, P, P, P, PoolDesc, P, I32, ctypes.c_float,
                                          I32, P, ctypes.c_size_t, P, P]
    ver = lib.pkv_paged_attn_verify
    # partition not a multiple of the 64-key tile; workspace missing
    assert ver(dummy, dummy, 2, 32, 8, 4, dummy, dummy, dummy, good, dummy, 8, 0.1, 100, ws, 1 << 20, dummy, None) == -2
    assert ver(dummy, dummy, 2, 32, 8, 4, dummy, dummy, dummy, good, dummy, 8, 0.1, 0, None, 0, dummy, None) == -5
    lib.pkv_verify_workspace_bytes.restype = ctypes.c_size_t
    lib.pkv_verify_workspace_bytes.argtypes = [I32] * 5
    # rows x heads x splits partials of d fp32 and their lse, about four splits
    assert lib.pkv_verify_workspace_bytes(256, 32, 128, 4096, 0) >= 256 * 32 * 4 * 129 * 4
    assert lib.pkv_verify_workspace_bytes(-1, 32, 128, 4096, 0) == 0
    # the automatic choice never cuts finer than 512 keys, and its workspace
    # is sized for exactly that (a context under 512 keys: one split)
    assert lib.pkv_verify_workspace_bytes(256, 32, 128, 4096, 0) == lib.pkv_verify_workspace_bytes(256, 32, 128, 4096, 512)
    assert lib.pkv_verify_workspace_bytes(16, 8, 64, 300, 0) == lib.pkv_verify_workspace_bytes(16, 8, 64, 300, 320)

    lib.pkv_qk_norm_rope_append.argtypes = [P, P, P, I32, I32, P, P, P, P, ctypes.c_float, ctypes.c_float,
                                            P, P, P, PoolDesc, P]
    pro = lib.pkv_qk_norm_rope_append
    assert pro(dummy, dummy, dummy, 4, 32, dummy, dummy, dummy, dummy, 1e-6, 1e6, dummy, dummy, dummy, good, None) != -1
    assert pro(dummy, dummy, dummy, 4, 32, dummy, dummy, dummy, dummy, 1e-6, 0.5, dummy, dummy, dummy, good, None) == -2
    assert pro(dummy, dummy, dummy, 4, 12, dummy, dummy, dummy, dummy, 1e-6, 1e6, dummy, dummy, dummy, good, None) == -2
    assert pro(None, dummy, dummy, 4, 32, dummy, dummy, dummy, dummy, 1e-6, 1e6, dummy, dummy, dummy, good, None) == -1

    lib.pkv_kv_append_cow.argtypes = [P, P, P, P, I32, P, I32, I32, P, P, I32, P, P, P, PoolDesc, P]
    cow = lib.pkv_kv_append_cow
    assert cow(dummy, dummy, dummy, dummy, 4, dummy, 2, 0, dummy, dummy, 3, dummy, dummy, dummy, good, None) == -2
    assert cow(dummy, dummy, dummy, dummy, 4, None, 2, 8, dummy, dummy, 3, dummy, dummy, dummy, good, None) == -1
    assert cow(None, None, None, None, 0, None, 2, 8, None, None, 0, None, None, None, good, None) == 0

    lib.pkv_paged_attn_chunked_prefill.argtypes = [P, P, I32, I32, I32, I32, P, P, P, PoolDesc, P,
                                                   I32, ctypes.c_float, P, P]
    pre = lib.pkv_paged_attn_chunked_prefill
    assert pre(dummy, dummy, 2, 32, 100, 64, None, dummy, dummy, good, dummy, 8, 0.1, dummy, None) == -1
    assert pre(dummy, dummy, 2, 32, -1, 64, dummy, dummy, dummy, good, dummy, 8, 0.1, dummy, None) == -2

    lib.pkv_split_k_combine.argtypes = [P, P, P, I32, I32, I32, I32, P, P, P]
    comb = lib.pkv_split_k_combine
    assert comb(dummy, dummy, dummy, 2, 32, 96, 4, dummy, None, None) == -3
    assert comb(dummy, dummy, dummy, 2, 32, 128, 0, dummy, None, None) == -2
    assert comb(None, dummy, dummy, 2, 32, 128, 4, dummy, None, None) == -1


def test_device_error_flags_rejects_null(lib):
    lib.pkv_device_error_flags.argtypes = [ctypes.c_void_p, ctypes.c_int]
    assert lib.pkv_device_error_flags(None, 0) == -1
